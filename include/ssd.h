/*
 * ssd.h -- C ABI of libssd: the batched verify + speculation-cache step of
 * Speculative Speculative Decoding (the Saguaro algorithm), hand-written CUDA
 * for B200 (sm_100a).
 *
 * Sources (cited by page title and section):
 *   [ZH] "Speculative Speculative Decoding", gist.science, Chinese edition,
 *        technical summary section 2 (Methodology): basic flow steps 1-4,
 *        challenge 1 (geometric fan-out), challenge 2 (Saguaro sampling),
 *        challenge 3 (fallback by batch size); section 1 (lossless SD).
 *   [NL] "Speculative Speculative Decoding", gist.science, Dutch edition,
 *        technical summary sections 2 and 3A / 3B / 3C.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * - Every pointer is a DEVICE pointer owned by the caller, unless a comment
 *   says otherwise.  The library never allocates, frees or synchronises; each
 *   call enqueues its kernels on `stream` (a cudaStream_t, NULL = legacy
 *   default stream) and returns at once.
 * - Logits are contiguous, row-major, of dtype SSD_DTYPE_BF16 (bf16 bit
 *   patterns) or SSD_DTYPE_FP32, and their base pointers are 16-byte aligned.
 *   Rows may start anywhere (V need not be a multiple of 8).
 * - Temperature T >= 0 and finite; T = 0 selects greedy verification (p and
 *   q one-hot at the lowest-index argmax of the raw logits).
 * - The return value reports host-detectable errors only (bad argument,
 *   alignment, workspace size, launch failure).  Data errors (NaN logits,
 *   tokens out of range, uniforms outside [0,1), a bad fan-out plan) are
 *   reported per row in `status` as SSD_ROW_* bits and never trap the GPU.
 * - A row whose status has a bit of SSD_ROW_INVALID set gets: n_accepted =
 *   -1, bonus = -1, out_tokens all -1, accept_prob and residual_mass NaN, its
 *   cache tokens -1, hit 0, slot -1, and fallback next_tokens.
 */
#ifndef SSD_H_
#define SSD_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum ssd_status {
  SSD_OK = 0,
  SSD_ERR_INVALID_ARG = 1,  /* a size, pointer or hyper-parameter is out of range */
  SSD_ERR_DTYPE = 2,        /* dtype is neither SSD_DTYPE_BF16 nor SSD_DTYPE_FP32 */
  SSD_ERR_ALIGNMENT = 3,    /* a logits or workspace pointer is not 16/256-byte aligned */
  SSD_ERR_WORKSPACE = 4,    /* workspace NULL or smaller than ssd_workspace_bytes() */
  SSD_ERR_CUDA = 5,         /* a kernel launch or attribute call failed */
  SSD_ERR_TIMEOUT = 6,      /* a device-side bounded wait gave up (ssd_read_device_error) */
  SSD_ERR_UNSUPPORTED = 7   /* V too large for the on-chip slice plan of this GPU */
} ssd_status;

typedef enum ssd_dtype { SSD_DTYPE_FP32 = 0, SSD_DTYPE_BF16 = 1 } ssd_dtype;

enum { SSD_FANOUT_GEOMETRIC = 0, SSD_FANOUT_UNIFORM = 1 };

/* Per-row status bits. */
#define SSD_ROW_NONFINITE 1       /* a NaN or +inf logit, or a vocab row that is all -inf */
#define SSD_ROW_BAD_TOKEN 2       /* a draft token outside [0, V) */
#define SSD_ROW_BAD_UNIFORM 4     /* a uniform outside [0, 1) or NaN */
#define SSD_ROW_ZERO_Q 8          /* informational: q'(d_j) == 0 at a draft position */
#define SSD_ROW_ZERO_RESIDUAL 16  /* informational: residual mass 0; bonus drawn from p */
#define SSD_ROW_NEAR_TIE 32       /* informational: a decision margin below 1e-5 */
#define SSD_ROW_BAD_PLAN 64       /* F entries negative, > V, or not summing to budget */
#define SSD_ROW_DEVICE_TIMEOUT 128 /* a bounded device wait gave up; outputs of the row are void */
#define SSD_ROW_INVALID (SSD_ROW_NONFINITE | SSD_ROW_BAD_TOKEN | SSD_ROW_BAD_UNIFORM | \
                         SSD_ROW_BAD_PLAN | SSD_ROW_DEVICE_TIMEOUT)

/* Limits of this build. */
#define SSD_MAX_K 32              /* draft length K */
#define SSD_MAX_BUDGET 512        /* fan-out branch budget (total cache keys per row) */

/*
 * Speculation cache of one batch ([ZH] section 2, basic flow step 3; [NL]
 * section 2, "speculation cache").  Keys are (accepted length k, bonus guess);
 * row b's keys for outcome k are tokens[b, offsets[b,k] : offsets[b,k+1]],
 * sorted by draft logit (descending, ties to the lower token id).  All
 * pointers are caller-owned device memory.
 */
typedef struct ssd_cache {
  int32_t* offsets;        /* [B, K+2]  out: prefix sums of F */
  int32_t* tokens;         /* [B, budget] out: bonus guesses, segment k = outcome k */
  const int32_t* payload;  /* [B, budget, K] in, or NULL: pre-speculated tokens per key */
  uint8_t* hit;            /* [B] out: 1 iff (n_accepted, bonus) is a key of the row */
  int32_t* slot;           /* [B] out: index of that key in tokens[b,:], -1 on a miss */
  int32_t* next_tokens;    /* [B, K] out: payload[b, slot, :] on a hit (-1 without a
                              payload); on a miss the fallback speculator's K random
                              tokens (ssd_cache_lookup) */
  uint64_t fallback_seed;  /* Philox key of the fallback stream */
} ssd_cache;

/*
 * ssd_fanout_plan -- geometric fan-out of the bonus-guess budget over the
 * accepted lengths k = 0..K ([ZH] section 2, challenge 1; [NL] section 3A:
 * the optimal split is a geometric series, more branches for the more likely
 * outcomes).  Reading: P(k) = alpha^k (1 - alpha) for k < K, P(K) = alpha^K,
 * F[b,k] = largest-remainder rounding of budget * P(k), ties to the smaller k.
 * mode SSD_FANOUT_UNIFORM is the uniform control: floor(budget/(K+1)) each,
 * remainder to the smallest k.  Computed in fp64 with no contraction.
 *   alpha [B] fp32 in [0, 1] (a row with alpha outside it gets F = 0 and
 *   -1 in F[b,0]); F [B, K+1] int32 out.  0 <= budget <= SSD_MAX_BUDGET.
 */
ssd_status ssd_fanout_plan(const float* alpha, int B, int K, int budget, int mode,
                           int32_t* F, void* stream);

/*
 * ssd_fanout_plan_power -- the power-law fan-out ([ZH] section 2, challenge
 * 1: the split follows the power law of the acceptance and is the solution of
 * a constrained optimisation; [NL] section 3A: a geometric series).  Reading:
 * when the hit rate of an outcome given F bonus guesses follows a power-law
 * curve 1 - c F^-beta, the budget-constrained optimum of the expected hit
 * rate puts F_k proportional to P(k)^gamma, gamma = 1 / (1 + beta): still
 * geometric in k, with ratio alpha^gamma.  gamma = gamma_eighths / 8,
 * gamma_eighths in 1..8 (8 is exactly ssd_fanout_plan's geometric plan).
 * alpha^gamma and (1 - alpha)^gamma are formed from three correctly rounded
 * square roots and gamma_eighths - 1 products; weights w_k = a^k c (k < K),
 * w_K = a^K; quotas budget * w_k / (w_0 + ... + w_K); largest remainder, ties
 * to the smaller k.  fp64, every operation rounded on its own.
 *   alpha [B] fp32 in [0, 1] (outside: F = 0 with -1 in F[b,0]); F [B, K+1]
 *   int32 out.  0 <= budget <= SSD_MAX_BUDGET.  Feed F to ssd_verify.
 */
ssd_status ssd_fanout_plan_power(const float* alpha, int B, int K, int budget, int gamma_eighths,
                                 int32_t* F, void* stream);

/*
 * ssd_alpha_update -- per-row acceptance estimate from history, the input of
 * the fan-out plans ([ZH] section 2, challenge 1: the split follows the
 * acceptance).  Reading: a_j is the expected acceptance of position j given
 * the drafts, so one step's estimate of the per-token acceptance is the mean
 * of accept_prob[b, 0..K-1], and alpha follows it by exponential smoothing:
 * alpha_out[b] = (1 - lambda) alpha[b] + lambda mean_j a_j (fp64, rounded
 * to fp32).  Rows with an SSD_ROW_INVALID bit, or a NaN a_j, keep alpha[b].
 *   alpha [B], accept_prob [B, K] (as ssd_verify writes it), status [B] in;
 *   alpha_out [B] out (may equal alpha).  0 <= lambda <= 1.
 */
ssd_status ssd_alpha_update(const float* alpha, const float* accept_prob, const int32_t* status, int B,
                            int K, double lambda, float* alpha_out, void* stream);

/*
 * ssd_fallback_bstar -- the fallback speculator by batch size ([ZH] section
 * 2, challenge 3; [NL] section 3C: a slow high-quality fallback for small
 * batches, a fast low-quality one -- n-gram or random tokens -- for large
 * ones, switching at a critical batch size b*).  HOST function, no device
 * work.  Reading: each row hits the cache with probability h; when any row
 * of a batch of b misses, the whole batch waits for the fallback, so a round
 * lasts L_target + (1 - h^b) L_fallback.  A hit, or a miss served by the
 * primary speculator, yields E_p = sum_{i=0..K} alpha^i tokens (expected
 * accepted drafts plus the bonus); a miss served by the fast one yields
 * E_fast.  The fast fallback is chosen for b when its expected tokens per
 * unit time are strictly higher.
 *   h: per-row hit probability (e.g. the mean of ssd_cache.hit); alpha:
 *   per-token acceptance; latencies in any one unit; choice: NULL or a HOST
 *   array of b_max bytes, choice[b-1] = 1 when batch size b takes the fast
 *   fallback.  Returns b* (the smallest such b), b_max + 1 when none does,
 *   -1 for arguments out of range.
 */
int ssd_fallback_bstar(double h, double alpha, int K, double L_target, double L_primary, double L_fast,
                       double E_fast, int b_max, uint8_t* choice);

/*
 * ssd_saguaro_reweight -- draft side ([ZH] section 2, challenge 2; [NL]
 * section 3B): for every (b, j < K), the top-F[b,j] tokens S_j of the draft
 * distribution q_j (by raw logit, ties to the lower id), Q_S = sum_{S_j} q_j,
 * Z_j = 1 - (1 - C) Q_S, and the log-normaliser of q_j; q'_j = w q_j / Z_j
 * with w = C on S_j and 1 elsewhere.  Optionally draws the draft token
 * d_j ~ q'_j by inverse CDF in token-id order with the uniform u_draft[b,j].
 *   draft_logits [B, K, V]; F [B, K+1]; 0 < C <= 1; budget <= min(V, SSD_MAX_BUDGET).
 *   guess_logits: NULL, or rows whose top-F[b,K] become segment K
 *     (full-acceptance guesses); row b starts at element b * guess_row_stride.
 *   u_draft [B, K] or NULL; draft_tokens_out [B, K] or NULL (needs u_draft).
 *   topf_tokens [B, budget] out (segment k at offsets[b,k]); offsets [B, K+2]
 *   out; Z [B, K] out; q_lse [B, K] out (natural log of sum_v exp(l(v)/T);
 *   the max logit when T = 0); status [B] out.
 *   workspace: ssd_workspace_bytes() bytes (see there).
 */
ssd_status ssd_saguaro_reweight(const void* draft_logits, int dtype, int B, int K, int V,
                                float T, const int32_t* F, float C, int budget,
                                const void* guess_logits, int64_t guess_row_stride,
                                const float* u_draft, int32_t* topf_tokens, int32_t* offsets,
                                float* Z, float* q_lse, int32_t* draft_tokens_out,
                                int32_t* status, void* workspace, size_t ws_bytes, void* stream);

/*
 * ssd_verify -- the fused verify + cache step: CTAs per (row, position,
 * vocabulary slice) stream that position's target and draft logits once.
 * Lossless verification ([ZH] sections 1-2; [NL] section 2) with Saguaro
 * reweighting: a_j = min(1, p_j(d_j) / q'_j(d_j)); position j is accepted iff
 * u[b,j] < a_j; n_accepted = k* = first rejected j, else K.  The bonus token
 * is drawn by inverse CDF (token-id order, strict >, uniform u[b,K]) from
 * r = max(0, p_{k*} - q'_{k*}) / R (from p_{k*} if R = 0), or from p_K after
 * full acceptance.  The fan-out plan is F when given; else, when alpha is
 * given, it is computed inside the kernel exactly as ssd_fanout_plan would
 * (alpha [B], fanout_mode); with neither there is no reweighting (C ignored)
 * and no cache.  With a cache, segment k < K is the top-F_k of q_k, segment K the
 * top-F_K of draft_next if given, else of the target row p_K; the lookup of
 * (k*, bonus) and the fallback follow ssd_cache_lookup.
 *   target_logits [B, K+1, V]; draft_logits [B, K, V]; draft_next [B, V] or NULL.
 *   draft_tokens [B, K]; uniforms [B, K+1] (columns < K: accept tests, column K:
 *   the bonus draw).  F [B, K+1] or NULL; 0 < C <= 1 when F is given.
 *   n_accepted [B], bonus [B], out_tokens [B, K+1] (accepted drafts, then the
 *   bonus, then -1), accept_prob [B, K] (a_j for every j), residual_mass [B]
 *   (R at k* < K, sum of p_K after full acceptance, 1 when T = 0), status [B].
 *   cache: NULL, or a host pointer to an ssd_cache of device pointers.
 *   workspace: as for ssd_saguaro_reweight.
 *   A build of the library with SSD_CLUSTER_VERIFY=1 runs the calls with
 *   bf16 logits, rows of a multiple of 8 tokens, T > 0 and budget <= 256 as
 *   one kernel of thread-block clusters (one cluster per row and position);
 *   arguments, outputs and error behaviour are the same.
 */
ssd_status ssd_verify(const void* target_logits, const void* draft_logits, const void* draft_next,
                      int dtype, int B, int K, int V, const int32_t* draft_tokens,
                      const float* uniforms, float T, const int32_t* F, const float* alpha,
                      int fanout_mode, float C, int budget,
                      int32_t* n_accepted, int32_t* bonus, int32_t* out_tokens,
                      float* accept_prob, float* residual_mass, const ssd_cache* cache,
                      int32_t* status, void* workspace, size_t ws_bytes, void* stream);

/*
 * ssd_verify_early_exit -- ssd_verify with the early-exit read schedule.
 * Lossless verification is a prefix test ([ZH] section 1, problem background,
 * and section 2, basic flow step 2: the drafts are checked in order and the
 * first rejection ends the accepted prefix), so the outcome (k*, the bonus,
 * the cache lookup) depends on the target rows p_0..p_{k*} and on p_K (the
 * source of segment K without draft_next, and of the bonus after full
 * acceptance) only.  The CTAs of position j (0 < j < K) are scheduled a lag
 * of rows after those of position j - 1, and a CTA does not read its slice of
 * p_j when an earlier position of its row is already known to be rejected.
 * Every draft row q_j is still read (the cache segments need them).
 *   Arguments and layouts: exactly as ssd_verify.  Outputs: as ssd_verify,
 *   except that accept_prob[b, j] is NaN for k* < j < K, and that a
 *   non-finite target row p_j or q'_j(d_j) = 0 at a position k* < j < K does
 *   not enter status (those rows are not part of the outcome; whether a CTA
 *   happened to read them never shows in the outputs).  The bytes it did not
 *   read are counted in the workspace (ssd_read_skipped_bytes).
 */
ssd_status ssd_verify_early_exit(const void* target_logits, const void* draft_logits, const void* draft_next,
                                 int dtype, int B, int K, int V, const int32_t* draft_tokens,
                                 const float* uniforms, float T, const int32_t* F, const float* alpha,
                                 int fanout_mode, float C, int budget,
                                 int32_t* n_accepted, int32_t* bonus, int32_t* out_tokens,
                                 float* accept_prob, float* residual_mass, const ssd_cache* cache,
                                 int32_t* status, void* workspace, size_t ws_bytes, void* stream);

/*
 * ssd_verify_noalloc -- ssd_verify with its scratch taken from a static
 * device buffer of this library instead of a caller-provided workspace.  The
 * pages describe no such call: it exists for callers that cannot allocate
 * device memory at the moment they verify -- a serving loop that handed
 * every byte of HBM to its KV cache at start-up, a host program with no
 * device allocator of its own, or code that must not let cudaMalloc/cudaFree
 * synchronise the device in the middle of a decode step.  It calls no
 * allocating function (no cudaMalloc, cudaFree or library allocation).
 *   Arguments, layouts, outputs and row status: exactly as ssd_verify, minus
 *   workspace and ws_bytes.
 *   Limit: the problem's ssd_workspace_bytes(B, K, V, dtype) must not exceed
 *   SSD_NOALLOC_MAX_WORKSPACE (16 MiB, enough for B=64, K=6, V=128256 bf16);
 *   larger problems return SSD_ERR_WORKSPACE before touching the device.
 *   First call on a device: looks up the buffer's device address
 *   (cudaGetSymbolAddress, with that device current); make that first call
 *   before any stream capture.  Every call then enqueues, on `stream` and
 *   ahead of its kernels, a cudaMemsetAsync that zeroes the part of the
 *   buffer holding this shape's arrival counters, decision words, epoch and
 *   error word (a few KB).  So a call never depends on the shape of the call
 *   before it, nor on whether that call timed out.  Device timeouts are
 *   reported through the rows' SSD_ROW_DEVICE_TIMEOUT bits only: the
 *   buffer's error word is cleared by the next call.
 *   The buffer is one per device, and the current device must own every
 *   pointer passed.  Calls that overlap on one device (two streams, or two
 *   host threads) share the buffer and race: serialise them.
 */
#define SSD_NOALLOC_MAX_WORKSPACE (16u << 20)
ssd_status ssd_verify_noalloc(const void* target_logits, const void* draft_logits, const void* draft_next,
                              int dtype, int B, int K, int V, const int32_t* draft_tokens,
                              const float* uniforms, float T, const int32_t* F, const float* alpha,
                              int fanout_mode, float C, int budget,
                              int32_t* n_accepted, int32_t* bonus, int32_t* out_tokens,
                              float* accept_prob, float* residual_mass, const ssd_cache* cache,
                              int32_t* status, void* stream);

/*
 * ssd_prespeculate -- pre-speculation of the cache payload ([ZH] section 2,
 * basic flow step 3: for each predicted verification outcome the draft
 * generates the following tokens in advance and stores them in the
 * speculation cache; [NL] section 2, "speculation cache").  For every cache
 * key s of row b the caller's draft model has produced logits for the K
 * positions after that key; this draws the K draft tokens of the key with
 * Saguaro sampling of the NEXT round ([ZH] challenge 2): d_i ~ q'_i, the
 * top-F_next[.,i] tokens of q_i down-weighted by C and renormalised, by
 * inverse CDF in token order with the caller's uniforms -- exactly
 * ssd_saguaro_reweight's draw on B * n_keys rows.
 *   key_logits [B, n_keys, K, V] (bf16 or fp32, 16-byte aligned);
 *   F_next [B * n_keys, K+1] the next round's plan per key (zeros with
 *   next_budget = 0 for plain sampling from q); 0 < C <= 1;
 *   uniforms [B, n_keys, K] in [0, 1); payload [B, n_keys, K] int32 out (the
 *   ssd_cache.payload layout when n_keys = budget); status [B * n_keys] out
 *   (SSD_ROW_* bits; an invalid key row gets -1 tokens).
 *   workspace: ssd_workspace_bytes(B * n_keys, K, V, dtype) bytes.
 *   T = 0 draws the argmax of each q_i.
 */
ssd_status ssd_prespeculate(const void* key_logits, int dtype, int B, int n_keys, int K, int V, float T,
                            const int32_t* F_next, float C, int next_budget, const float* uniforms,
                            int32_t* payload, int32_t* status, void* workspace, size_t ws_bytes,
                            void* stream);

/*
 * ssd_cache_build -- pack per-outcome guess lists into the cache layout
 * ([ZH] section 2, basic flow step 3).  offsets[b] = prefix sums of F[b];
 * tokens[b, offsets[b,k] + i] = topf_tokens[b, offsets[b,k] + i] for k < K
 * (the layout ssd_saguaro_reweight writes), and for k = K from guess_K[b, i]
 * when guess_K is given (else from topf_tokens as well).  i < F[b,k].
 *   F [B, K+1]; topf_tokens [B, budget]; guess_K [B, budget] or NULL;
 *   offsets [B, K+2] out; tokens [B, budget] out.
 */
ssd_status ssd_cache_build(const int32_t* F, const int32_t* topf_tokens, const int32_t* guess_K,
                           int B, int K, int budget, int32_t* offsets, int32_t* tokens,
                           void* stream);

/*
 * ssd_cache_lookup -- the outcome (k[b], bonus[b]) against the cache ([ZH]
 * section 2, basic flow step 4: a hit returns the pre-speculated tokens at
 * once; challenge 3 / [NL] section 3C: on a miss the fallback speculator, here
 * K uniformly random tokens).  hit[b] = 1 iff bonus[b] is in segment k[b];
 * slot[b] = its index in tokens[b,:], else -1.  next_tokens[b,i] =
 * payload[b, slot, i] on a hit (-1 without a payload); on a miss
 * floor(x * V / 2^32), x = first word of Philox4x32-10 (Salmon et al., SC'11)
 * with key = fallback_seed and counter (b, i, 2, 0).
 *   offsets [B, K+2]; tokens [B, budget]; k [B]; bonus [B]; payload [B, budget, K]
 *   or NULL; hit [B], slot [B], next_tokens [B, K] out.
 */
ssd_status ssd_cache_lookup(const int32_t* offsets, const int32_t* tokens, int B, int K,
                            int budget, const int32_t* k, const int32_t* bonus,
                            const int32_t* payload, uint64_t fallback_seed, int V,
                            uint8_t* hit, int32_t* slot, int32_t* next_tokens, void* stream);

/* Workspace size in bytes for ssd_verify / ssd_saguaro_reweight at
 * (B, K, V, dtype).  The workspace holds per-slice and per-(row, position)
 * partial results, per-row states, per-row decision words tagged with a call
 * epoch, then arrival counters and one device error word.  It must be 256-byte aligned and zero-filled before its first use;
 * each completed call leaves the counters zero again, so it can be reused by
 * the next call on the same stream (calls that overlap on the GPU must not
 * share one).  0 for invalid sizes. */
size_t ssd_workspace_bytes(int B, int K, int V, int dtype);

/* Reads and clears the device error word of a workspace laid out for
 * (B, K, V, dtype), synchronising `stream`: *out = SSD_OK, or SSD_ERR_TIMEOUT
 * when a bounded device wait of an earlier call gave up.  After a timeout the
 * workspace's counters may be left non-zero: zero-fill it again before its
 * next use.  Not for the hot path. */
ssd_status ssd_read_device_error(void* workspace, int B, int K, int V, int dtype, void* stream,
                                 int32_t* out);

/* Reads and clears the workspace's count of target-logit bytes that calls of
 * ssd_verify_early_exit on it did not read (B, K, V, dtype as laid out),
 * synchronising `stream`.  A measurement helper, not for the hot path. */
ssd_status ssd_read_skipped_bytes(void* workspace, int B, int K, int V, int dtype, void* stream,
                                  uint64_t* out);

const char* ssd_status_string(ssd_status s);
const char* ssd_version(void);

#ifdef __cplusplus
}
#endif

#endif /* SSD_H_ */
