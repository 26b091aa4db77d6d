/*
 * dspark.h -- C ABI of the DSpark per-round token path on B200 (sm_100a).
 *
 * One speculative-decoding round for a batch of B requests with draft block
 * size G over a V-token vocabulary, in four calls:
 *   dspark_draft_markov  semi-autoregressive drafting with the Markov head
 *   dspark_confidence    linear confidence head and prefix survival
 *   dspark_schedule      Algorithm-1 hardware-aware prefix scheduler
 *   dspark_verify        exact rejection-sampling verification
 *
 * Sources (web pages about arXiv:2607.05147, "DSpark: Confidence-Scheduled
 * Speculative Decoding with Semi-Autoregressive Generation"), cited by tag:
 *   [PL] paperlayer.ai section-by-section summary (§2 Background, §3.1
 *        Semi-autoregressive generation, §3.2 Confidence-scheduled
 *        verification, Appendix A counterexample);
 *   [KB] menfem.com knowledge-base entry ("Key Contributions",
 *        "Methodology");
 *   [WK] llm-wiki.hwlabs.dev study 116 (draft-generation figure of the
 *        Markov-head section; confidence-scheduling section).
 *
 * Conventions shared by every call
 * --------------------------------
 * - Every array pointer is a DEVICE pointer owned by the caller; the library
 *   keeps no pointer past the call's return, never allocates device or host
 *   memory, and never synchronises (except dspark_get_device_status).  Work
 *   is enqueued on `stream` (a cudaStream_t; NULL = the legacy default
 *   stream), so every call may be captured in a CUDA graph.
 * - Arrays are dense, row-major, with the shapes given; "dtype" arrays hold
 *   DSPARK_F32 (fp32) or DSPARK_BF16 (bf16 bit patterns) elements.
 * - Host-detectable errors (bad sizes, null pointers, short workspace, CUDA
 *   launch failures) return a non-zero dspark_status before or instead of
 *   enqueuing work.  Data errors that only the device can see (a token id
 *   outside [0, V), an admitted length outside [0, G], a negative or NaN
 *   temperature) are clamped to the valid range and recorded as bits of a
 *   status word at the start of the caller's workspace; read them with
 *   dspark_get_device_status.  No call traps, asserts or spins unbounded on
 *   the device.
 * - A workspace is caller-allocated device memory of at least the size the
 *   matching *_workspace_size query returns, aligned to 256 bytes.  One
 *   buffer of the largest size may serve every call of a round.  Workspace
 *   contents need no initialisation except the status word (see
 *   dspark_clear_device_status); calls that share a workspace must not run
 *   concurrently.
 * - Limits checked on the host: 1 <= B <= 4096, 1 <= G <= 16,
 *   2 <= V <= 2^20, 1 <= r <= 512 (a multiple of 16 for bf16), 1 <= d <= 65536,
 *   B*G <= 16384 for the scheduler, 1 <= P <= 64 profile knots.  For bf16
 *   rounds V is a multiple of 8 and the bf16 arrays (L, U, Wt, Tlog) start on
 *   16-byte boundaries (TMA and vector loads); otherwise DSPARK_ERR_INVALID_ARG.
 */
#ifndef DSPARK_H
#define DSPARK_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    DSPARK_OK = 0,
    DSPARK_ERR_INVALID_ARG = 1,      /* a size, pointer, mode or dtype is out of range */
    DSPARK_ERR_UNSUPPORTED_DTYPE = 2,
    DSPARK_ERR_WORKSPACE = 3,        /* workspace missing, short or misaligned */
    DSPARK_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed */
    DSPARK_ERR_TIMEOUT = 5           /* a bounded device wait gave up */
} dspark_status;

typedef enum { DSPARK_F32 = 0, DSPARK_BF16 = 1 } dspark_dtype;

typedef enum {
    DSPARK_SCHED_ALL = 0,               /* verify every drafted position */
    DSPARK_SCHED_GREEDY_EARLY_STOP = 1, /* Algorithm 1 */
    DSPARK_SCHED_GLOBAL_ARGMAX = 2,     /* variant: offline search, no early stop */
    DSPARK_SCHED_THRESHOLD = 3,         /* variant: static survival threshold (dspark_schedule_threshold) */
    DSPARK_SCHED_TOPK = 4               /* variant: dynamic top-K of the production scheduler (dspark_schedule_topk) */
} dspark_sched_mode;

/* Bits of the device status word. */
#define DSPARK_DEV_TOKEN_RANGE 0x1u  /* a token id outside [0, V) was clamped */
#define DSPARK_DEV_ELL_RANGE 0x2u    /* an admitted length outside [0, G] was clamped */
#define DSPARK_DEV_BAD_TEMP 0x4u     /* a temperature < 0 or NaN was treated as 0 */
#define DSPARK_DEV_TIMEOUT 0x8u      /* a bounded device wait ran out */
#define DSPARK_DEV_BAD_VALUE 0x10u   /* calibration: a non-finite logit, or a grid entry that is no temperature */

/* Library version and the build's target (a string such as "sm_100a"). */
const char *dspark_version(void);

/* ------------------------------------------------------------------------ */
/* Stage 1: semi-autoregressive drafting with the Markov head.
 * [PL] §3.1: the parallel backbone gives all G draft logit rows in one pass;
 * a lightweight sequential module then samples left to right, each position
 * conditioned on the previously sampled token through a low-rank transition
 * matrix.  [KB] Methodology: rank-256 factorisation.  [WK] draft-generation
 * figure: final logits L[i] + Delta[i], then the draft token is sampled.
 *
 * For i = 1..G in order (x_0 = x0[b], the last committed token):
 *   y = L[b,i,:] + Delta_i[b,:],  Delta_i[b,v] = sum_k U[x_{i-1},k] * Wt[v,k]
 *   z = y / T_b,  m = max z,  Z = sum_v exp(z_v - m)
 *   x_i = smallest v with u_draft[b,i] < sum_{j<=v} exp(z_j - m) / Z
 *   (T_b = 0: x_i = argmax y, lowest index on ties).
 * Inputs:  L [B,G,V] dtype, U [V,r] dtype, Wt [V,r] dtype (the transition
 *          factor W stored transposed: row v is column v of W), x0 [B] int32,
 *          temp [B] f32 (>= 0), u_draft [B,G] f32 in [0,1).
 * Outputs: x_out [B,G] int32; pd_x_out [B,G] f32 = p_d(x_i) (1 for T = 0);
 *          rowmax_out [B,G] f32 = max_v y_v (before the temperature);
 *          rowsum_out [B,G] f32 = Z (1 for T = 0).
 * rowmax/rowsum are what dspark_verify needs to rebuild p_d at a rejection. */
size_t dspark_draft_workspace_size(int B, int G, int V, int r, int dtype);
dspark_status dspark_draft_markov(const void *L, const void *U, const void *Wt,
                                  const int32_t *x0, const float *temp,
                                  const float *u_draft, int B, int G, int V, int r,
                                  int dtype, void *ws, size_t ws_bytes, int32_t *x_out,
                                  float *pd_x_out, float *rowmax_out, float *rowsum_out,
                                  void *stream);

/* ------------------------------------------------------------------------ */
/* Stage 2: confidence head and prefix survival.
 * [KB] Key Contributions: a lightweight linear confidence head emits a
 * per-position survival probability.  [PL] §3.2: it estimates each draft
 * token's conditional survival; cumulative products give prefix survival,
 * calibrated left to right by sequential temperature scaling.
 *   c[b,i] = sigmoid((w . h[b,i,:] + bias) / tau[i]),  S[b,i] = prod_{j<=i} c[b,j].
 * Inputs:  h [B,G,d] dtype, w [d] dtype, bias, tau [G] f32 or NULL (all 1).
 * Outputs: c_out [B,G] f32, S_out [B,G] f32 (non-increasing along i).
 * Needs no workspace. */
dspark_status dspark_confidence(const void *h, const void *w, float bias, const float *tau,
                                int B, int G, int d, int dtype, float *c_out, float *S_out,
                                void *stream);

/* ------------------------------------------------------------------------ */
/* Stage 3: Algorithm 1, the hardware-aware prefix scheduler.
 * [KB] Key Contributions: greedy global sort of candidate tokens by
 * cumulative survival, incremental batch admission with early stopping that
 * keeps admissions causal.  [PL] Appendix A: stop as soon as the objective
 * drops (Theta_{n+1} < Theta_n); admitting token k may use only information
 * available before x_k is sampled.
 *   Candidates (b, i) are laid out position-major (idx = i*B + b) and sorted
 *   by S descending, ties by idx, so every request's admitted set is a prefix.
 *   V_0 = B, Theta_n = V_n / t(n); candidate n+1 is admitted unless
 *   (V_n + S_(n+1)) * t(n) < V_n * t(n+1) (evaluated in fp64); admission
 *   also ends at `budget` (< 0: none) or when all B*G are admitted.
 *   t(n) is piecewise linear through the P knots (knots_n[j], knots_t[j]),
 *   knots_n[0] = 0 and strictly increasing, continued past the last knot
 *   with the last segment's slope (constant when P = 1); knots_t > 0.
 *   mode DSPARK_SCHED_GLOBAL_ARGMAX (a scheduler variant, the offline global
 *   search of [PL] Appendix A): the admitted count is the n in 0..budget
 *   that maximises Theta_n (the lowest such n); it may look past a drop of
 *   Theta, so with confidences that depend on drawn tokens it is not
 *   lossless ([PL] Appendix A's counterexample).
 * Inputs:  S [B,G] f32, knots_n [P] int32, knots_t [P] f64 (device arrays),
 *          budget, mode (DSPARK_SCHED_ALL, _GREEDY_EARLY_STOP or
 *          _GLOBAL_ARGMAX; anything else is DSPARK_ERR_INVALID_ARG).
 * Outputs: ell_out [B] int32 admitted prefix length per request;
 *          n_adm_out [1] int32; theta_out [1] f64 = Theta at n_adm;
 *          order_out [B*G] int32 sorted candidate indices, or NULL. */
size_t dspark_schedule_workspace_size(int B, int G);
dspark_status dspark_schedule(const float *S, int B, int G, const int32_t *knots_n,
                              const double *knots_t, int P, int budget, int mode, void *ws,
                              size_t ws_bytes, int32_t *ell_out, int32_t *n_adm_out,
                              double *theta_out, int32_t *order_out, void *stream);

/* Scheduler variant: static-threshold pruning.  [KB] Key Contributions ranks
 * candidates by cumulative survival; this variant admits, in the same stable
 * order (S descending, ties by position-major index), every candidate with
 * S >= threshold, at most `budget` (< 0: none).  No profile and no objective:
 * the cut depends on the survival level alone, so a request's admitted
 * positions are a prefix whenever its S is non-increasing (as the confidence
 * stage's cumulative products are).
 * Inputs:  S [B,G] f32, threshold, budget; same limits and workspace as
 *          dspark_schedule.
 * Outputs: ell_out [B] int32, n_adm_out [1] int32, order_out [B*G] int32 or
 *          NULL. */
dspark_status dspark_schedule_threshold(const float *S, int B, int G, float threshold, int budget, void *ws,
                                        size_t ws_bytes, int32_t *ell_out, int32_t *n_adm_out,
                                        int32_t *order_out, void *stream);

/* Scheduler variant: the production scheduler's dynamic top-K.  [PL] §5.2
 * Production Scheduler: the scheduler runs asynchronously; the capacity limit
 * comes from historical predictions and the current candidates are ranked by
 * their latest cumulative confidence; the top-K selection keeps the
 * confidence ordering and hides the scheduling latency, and the capacity's
 * global search copes with irregular hardware-capacity curves.  This call is
 * the selection: it admits the first K candidates of the same stable order as
 * dspark_schedule, K = *capacity clamped to [0, B*G], at most `budget` (< 0:
 * none).  `capacity` is a DEVICE int32, typically the n_adm_out of a
 * dspark_schedule call in mode DSPARK_SCHED_GLOBAL_ARGMAX on the previous
 * round's survivals, enqueued on another stream while this round drafts; the
 * count is read when the kernel runs, so one captured graph serves every
 * capacity.  A negative capacity admits none and sets DSPARK_DEV_ELL_RANGE in
 * the workspace's status word.
 * Inputs:  S [B,G] f32, capacity [1] int32 (device), budget; limits and
 *          workspace as dspark_schedule.
 * Outputs: ell_out [B] int32, n_adm_out [1] int32, order_out [B*G] int32 or
 *          NULL. */
dspark_status dspark_schedule_topk(const float *S, int B, int G, const int32_t *capacity, int budget, void *ws,
                                   size_t ws_bytes, int32_t *ell_out, int32_t *n_adm_out, int32_t *order_out,
                                   void *stream);

/* ------------------------------------------------------------------------ */
/* Stage 4: exact rejection-sampling verification.
 * [KB] Methodology: x_k is accepted with probability min(1, p_t(x_k) /
 * p_d(x_k)); the first rejection discards every later token.  [PL] §2:
 * verification runs left to right and keeps the longest consistent prefix.
 * [PL] Appendix A: with nothing admitted the target draws a fresh token.
 *   p_t = softmax(Tlog[b,k,:] / T_b).  For k = 1..ell_b: accept x_k iff
 *   u_accept[b,k] < p_t(x_k) / pd_x[b,k]; A_b = leading accepts.
 *   If A_b < ell_b: y ~ normalised max(0, p_t - p_d) at k* = A_b + 1, with
 *   p_d rebuilt from L, U, Wt, rowmax, rowsum (an all-zero residual falls
 *   back to p_t).  Else y ~ p_t at row ell_b + 1 (the bonus token).  Draws
 *   are inverse-CDF with u_final[b].  T_b = 0: accept iff argmax Tlog[b,k]
 *   = x_k, and y = argmax Tlog[b, A_b + 1].
 * Inputs:  Tlog [B,G+1,V] dtype (row k verifies x_k; row G+1 is the bonus
 *          row), L, U, Wt, x0 as for drafting, x/pd_x/rowmax/rowsum from
 *          dspark_draft_markov, temp [B], u_accept [B,G], u_final [B] f32,
 *          ell [B] int32 from dspark_schedule.
 * Outputs: acc_out [B] int32 = A_b; tokens_out [B,G+1] int32 = x_1..x_A, y,
 *          then -1; nout_out [B] int32 = A_b + 1; pt_x_out [B,G] f32 =
 *          p_t(x_k) for k <= ell_b (1/0 for T = 0, match/no match; -1
 *          elsewhere), or NULL. */
size_t dspark_verify_workspace_size(int B, int G, int V, int r, int dtype);
dspark_status dspark_verify(const void *Tlog, const void *L, const void *U, const void *Wt,
                            const int32_t *x0, const int32_t *x, const float *pd_x,
                            const float *rowmax, const float *rowsum, const float *temp,
                            const float *u_accept, const float *u_final, const int32_t *ell,
                            int B, int G, int V, int r, int dtype, void *ws, size_t ws_bytes,
                            int32_t *acc_out, int32_t *tokens_out, int32_t *nout_out,
                            float *pt_x_out, void *stream);

/* ------------------------------------------------------------------------ */
/* The RNN sequential head.  [PL] §3.1: the sequential stage conditions each
 * position on the tokens sampled before it; besides the Markov head's
 * low-rank transition matrix it names an RNN head whose recurrent state
 * summarises the whole in-block prefix.  [KB] Key Contributions: the two
 * variants (first-order dependency by a low-rank factorisation; the full
 * within-block history).  The pages give no equations; the reading here is
 * the plainest recurrence over the Markov head's factors: a state of size r,
 *   h_1 = tanh(U[x_0]),  h_k = tanh(h_{k-1} Arec + U[x_{k-1}]),
 *   Delta_k = h_k W  (Delta_k[v] = sum_c h_k[c] * Wt[v,c]),
 * with everything else as in dspark_draft_markov / dspark_verify.
 *
 * dspark_draft_rnn: as dspark_draft_markov, plus Arec [r,r] bf16 (row q,
 *   column c: the weight from state q to state c) and the output
 *   H_out [B,G,r] f32: H_out[b,k-1,:] = h_k, the state that biased position k
 *   (verification rebuilds p_d from it).  bf16 only (DSPARK_ERR_UNSUPPORTED_DTYPE
 *   otherwise), r <= 256, H_out 16-byte aligned; same workspace size.
 *   The state is computed in fp32 and enters the tensor-core product as two
 *   bf16 parts (high + low, about 2^-17 relative).
 * dspark_verify_rnn: as dspark_verify with the states H [B,G,r] f32 from
 *   dspark_draft_rnn in place of U and x0 (the residual at a rejection
 *   rebuilds p_d from L + h_k W).  Same limits as dspark_draft_rnn. */
dspark_status dspark_draft_rnn(const void *L, const void *U, const void *Arec, const void *Wt,
                               const int32_t *x0, const float *temp, const float *u_draft, int B,
                               int G, int V, int r, int dtype, void *ws, size_t ws_bytes,
                               int32_t *x_out, float *pd_x_out, float *rowmax_out,
                               float *rowsum_out, float *H_out, void *stream);
dspark_status dspark_verify_rnn(const void *Tlog, const void *L, const float *H, const void *Wt,
                                const int32_t *x, const float *pd_x, const float *rowmax,
                                const float *rowsum, const float *temp, const float *u_accept,
                                const float *u_final, const int32_t *ell, int B, int G, int V,
                                int r, int dtype, void *ws, size_t ws_bytes, int32_t *acc_out,
                                int32_t *tokens_out, int32_t *nout_out, float *pt_x_out,
                                void *stream);

/* ------------------------------------------------------------------------ */
/* Target rows from host memory.  [PL] §2: the target model checks the drafted
 * tokens in one forward pass; [KB] Key Contributions: the scheduler prunes
 * low-confidence tokens from verification.  The target forward therefore
 * yields rows only for the admitted positions: of Tlog [B,G+1,V] a round
 * needs rows 0..ell_b of request b (ell_b verified positions, then the row of
 * the bonus or residual draw), and dspark_verify / dspark_verify_rnn read no
 * other row.  This call enqueues one kernel that copies exactly those rows
 * from page-locked host memory into the device buffer of the same layout,
 * reading ell on the device (e.g. dspark_schedule's ell_out, earlier on the
 * same stream), so a round fed from the host needs no host round trip
 * between scheduling and verification and stays graph-capturable.  The other
 * rows of the device buffer are left as they are.  Nothing is allocated or
 * synchronised.
 * Inputs:  Tlog_host [B,G+1,V] dtype in page-locked host memory that the
 *          device can address (cudaHostAlloc / cudaMallocHost memory under
 *          unified addressing); ell [B] int32 (device), each clamped to
 *          [0, G] when read.
 * Outputs: Tlog_dev [B,G+1,V] dtype (device memory).
 * Errors:  DSPARK_ERR_UNSUPPORTED_DTYPE; DSPARK_ERR_INVALID_ARG for a null
 *          pointer, B outside [1, 4096], G outside [1, 16], V outside
 *          [1, 2^24], a source that is not device-addressable page-locked host
 *          memory or a destination that is not device memory (nothing is
 *          enqueued); DSPARK_ERR_CUDA if the launch fails.  The caller
 *          guarantees that both buffers hold B*(G+1)*V elements. */
dspark_status dspark_gather_admitted_targets(const void *Tlog_host, void *Tlog_dev, const int32_t *ell, int B,
                                             int G, int V, int dtype, void *stream);

/* ------------------------------------------------------------------------ */
/* Drafting without a workspace, for callers that cannot allocate device
 * memory when they draft: e.g. a plugin of an inference engine that receives
 * only its inputs and outputs at enqueue time (the engine planned all memory
 * ahead and offers no allocator), or a latency-critical serving loop that must
 * not call cudaMalloc, which can synchronise the whole device.  The paper has
 * no counterpart to this entry point; it is an engineering variant of
 * dspark_draft_markov with identical arguments and results, minus the
 * workspace.
 *
 * Its scratch lives in a file-scope device array of
 * dspark_draft_noalloc_max_scratch() bytes (8 MiB) that every GPU which loads
 * this library holds until the process exits.  Rounds whose drafting
 * workspace (dspark_draft_workspace_size) would exceed that size are rejected
 * with DSPARK_ERR_WORKSPACE before any work is enqueued; the headline shape
 * B = 256, G = 5, V = 129280, r = 256 needs 4,530,432 bytes.  No call
 * allocates: no cudaMalloc, cudaFree or allocating library routine.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it; make that first call before any stream
 * capture.  Every call reuses the same array, which keeps the previous call's
 * contents: the call clears the status word it needs to start at zero, and
 * the rest is written before it is read.  Calls that may overlap on the GPU
 * (other streams, other host threads) race on the array and must be
 * serialised by the caller.  Device-side data errors and a bounded wait
 * that ran out are clamped or abandoned as in dspark_draft_markov and
 * recorded in the array's status word, which the call clears first:
 * dspark_draft_noalloc_device_status synchronises `stream` and copies that
 * word (the DSPARK_DEV_* bits of the last call enqueued on `stream`) to
 * *status_out.  After DSPARK_DEV_TIMEOUT the outputs are not valid. */
size_t dspark_draft_noalloc_max_scratch(void);
dspark_status dspark_draft_noalloc_device_status(void *stream, uint32_t *status_out);
dspark_status dspark_draft_markov_noalloc(const void *L, const void *U, const void *Wt,
                                          const int32_t *x0, const float *temp,
                                          const float *u_draft, int B, int G, int V, int r,
                                          int dtype, int32_t *x_out, float *pd_x_out,
                                          float *rowmax_out, float *rowsum_out, void *stream);

/* ------------------------------------------------------------------------ */
/* ------------------------------------------------------------------------ */
/* Confidence calibration: sequential temperature scaling (STS).
 * [PL] §3.2: STS calibrates the cumulative prefix-survival probabilities left
 * to right, minimising the expected calibration error (ECE) of the running
 * products of the per-position scores while keeping their ordering.  [KB]
 * Key Contributions (post-hoc, left to right) and Results (ECE 3-8 % raw,
 * about 1 % after STS).  The fitted tau is what dspark_confidence takes.
 *   Labels: y[n,i] = 1 if acc[n] >= i (i = 1..G): the first i draft tokens of
 *   block n were accepted (acc = the accepted counts of blocks verified at
 *   full length, e.g. dspark_verify's acc_out under DSPARK_SCHED_ALL).
 *   Scores: S[n,i] = S[n,i-1] * sigmoid(z[n,i] / tau_i), S[n,0] = 1.
 *   ECE(s, y) = sum over M equal-width bins of |sum_{n in bin} (y_n - s_n)| / N,
 *   bin(s) = min(M - 1, floor(s * M)).
 *   Fit: for i = 1..G in turn (earlier tau fixed), tau_i = the first entry of
 *   tau_grid with the least ECE(S[:,i], y[:,i]).  A grid entry that is not a
 *   positive finite number has ECE +inf (and sets DSPARK_DEV_BAD_VALUE).
 *   All arithmetic in fp64 (scores, bins, sums); the per-bin sums run in a
 *   fixed order, so the result is deterministic.
 * Inputs:  z [N,G] f32 head logits (w . h + bias, before any temperature),
 *          acc [N] int32 in [0, G] (others: DSPARK_DEV_ELL_RANGE, labels as
 *          defined), tau_grid [K] f32, n_bins M.
 * Outputs: tau_out [G] f32; ece_raw_out [G] f64 (tau = 1), ece_fit_out [G]
 *          f64, ece_all_out [G,K] f64 (every candidate), S_out [N,G] f32 (the
 *          fitted survivals rounded to fp32); the last four may be NULL.
 * Limits:  1 <= N <= 2^24, 1 <= G <= 16, 1 <= K <= 4096, 1 <= M <= 32.
 * Enqueues a 4-byte memset and G kernel launches. */
size_t dspark_sts_workspace_size(int N, int G, int K, int n_bins);
dspark_status dspark_sts_fit(const float *z, const int32_t *acc, const float *tau_grid, int N, int G, int K,
                             int n_bins, void *ws, size_t ws_bytes, float *tau_out, double *ece_raw_out,
                             double *ece_fit_out, double *ece_all_out, float *S_out, void *stream);

/* ROC-AUC of the prefix survivals against the same labels ([KB] Results
 * reports the raw confidence's ROC-AUC): for each position i, over every pair
 * of a positive (acc[p] >= i) and a negative sample, 2 when the positive's
 * S is larger, 1 on a tie, 0 otherwise (NaN scores compare false).
 * Inputs:  S [N,G] f32, acc [N] int32.
 * Outputs: twice_out [G] uint64 = the pair total; pairs_out [G] uint64 =
 *          positives * negatives; AUC_i = twice_out[i] / (2 * pairs_out[i]).
 *          Exact integers.  Needs no workspace; limits as dspark_sts_fit. */
dspark_status dspark_survival_auc(const float *S, const int32_t *acc, int N, int G, uint64_t *twice_out,
                                  uint64_t *pairs_out, void *stream);

/* Device status word of a workspace: dspark_get_device_status synchronises
 * `stream`, then copies the word to *status_out (0 = no data error since the
 * last clear).  dspark_clear_device_status enqueues a reset of the word and
 * of the near-tie counts below. */
dspark_status dspark_get_device_status(const void *ws, void *stream, uint32_t *status_out);
dspark_status dspark_clear_device_status(void *ws, void *stream);

/* Near-tie counts of a workspace since its last clear: the sampled decisions
 * whose uniform fell within 1e-5 of the threshold that would flip them, as
 * the kernels evaluate them in fp32 -- a draw's uniform within 1e-5 (CDF
 * units) of an edge of the chosen token's interval, or one that rounding left
 * past the row's mass (drafting: *draft_out; the bonus, fresh and residual
 * draws of verification: *verify_out), and an accept test with
 * |u - p_t(x)/p_d(x)| < 1e-5 among the tests that decided the accepted count
 * (*verify_out).  Such a decision can differ from an exact computation of
 * the same round; argmax decisions (temperature 0) are not counted.
 * Synchronises `stream`. */
dspark_status dspark_get_near_ties(const void *ws, void *stream, uint32_t *draft_out, uint32_t *verify_out);

/* Diagnostics: y[i] = 2^x[i] by the FMA-pipe polynomial that shares the
 * exponentials of the verification row pass with the special-function unit
 * (x = n + f, n = rint(x), f in [-1/2, 1/2]; 2^f from a degree-5 polynomial;
 * 2^n added to the exponent bits).  Relative error within 4e-7 of 2^x for
 * -125 <= x <= 0; arguments below -125 give 2^-125.  x, y: device arrays of n
 * floats (n >= 0), enqueued on `stream`.  DSPARK_ERR_INVALID_ARG for a null
 * pointer with n > 0 or a negative n. */
dspark_status dspark_exp2_fma(const float *x, float *y, int n, void *stream);

#ifdef __cplusplus
}
#endif

#endif /* DSPARK_H */
