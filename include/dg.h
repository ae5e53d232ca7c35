/*
 * dg.h -- C ABI of the B200 (sm_100a) sampler library for block-parallel
 * uniform-noise discrete diffusion (DiffusionGemma-style denoising).
 *
 * Pages cited: DiffusionGemma Technical Report, hyper.ai paper summary,
 *   section "Method"  -- forward probability path
 *       P(X_t = x_t | X_0 = x_0) = prod_i [kappa_t delta(x_t^i, x_0^i) + (1 - kappa_t)/V],
 *     the schedule kappa (monotone, kappa_0 = 1, kappa_1 = 0), the Step
 *     reverse transition, the per-iteration update
 *       p0 = Softmax(L_t / tau_t),  z = FFW(p0 E),  x_{t-dt} ~ Step(x_t, p0),
 *     the sampler paragraph (entropy-ordered acceptance under an error
 *     tolerance with uniform re-noising, tau annealed linearly 0.8 -> 0.4,
 *     adaptive stopping), and the canvas loss
 *       L = -sum_{i=1..C} log p(x_0^i | x_t, z_t, H);
 *   section "Dataset" -- training sequences of P prompt tokens + K canvases of
 *     C tokens; the decoder loss on one canvas per sequence chosen uniformly;
 *     the self-conditioning state used for half of the batch, zero otherwise.
 *
 * Conventions shared by every entry point
 *   - Every function returns an int status (dg_status).  On failure nothing
 *     has been launched, and dg_last_error() (thread-local) says why.
 *   - Device buffers are owned by the caller and are never freed or kept by
 *     the library.  The library allocates no device memory: scratch comes
 *     from a caller workspace sized by the matching *_workspace_size query.
 *     A workspace must be zero-filled before its first use, and again before
 *     it is reused for a call of a different shape (rows, V, n_seq): the
 *     layout inside it depends on the shape.  Every call that returns DG_OK
 *     leaves it ready for the next call of the same shape (its counters back
 *     at zero, the call counter that tags the logits pass's records
 *     advanced), so one workspace serves any number of successive same-shape
 *     calls on one stream.  Two calls that run at the same time need two
 *     workspaces.
 *   - Per-canvas scalars (t, dt, inv_tau) are HOST arrays, read during the
 *     call; everything else named "device" is device memory.
 *   - All work is enqueued asynchronously on `stream` (a cudaStream_t;
 *     NULL = the legacy default stream).  Arguments are checked before any
 *     launch.  Device-side waits are bounded: one that expires sets a device
 *     error word read (and cleared) by dg_device_error(); re-zero the
 *     workspace after such an error.
 *   - Logits rows: element (r, v) lives at logits + r*ld + v (elements), the
 *     base is 16-byte aligned and ld*sizeof(element) is a multiple of 16.
 *     Logits must be finite or -inf (a masked token); NaN is not supported.
 *   - Random numbers: Philox4x32-10 (Salmon et al., SC'11) with key
 *     (seed & 0xffffffff, seed >> 32); counter word 3 names the use:
 *       0 token Gumbel     (v >> 2, row, step, 0), word v & 3
 *       1 Step             (0, row, step, 1): word 0 branch, word 1 token
 *       2 forward noise    (j, b, 0, 2): word 0 keep, word 1 token
 *       3 loss canvas      (0, b, 0, 3): word 0
 *       4 chunk Gumbel     (c >> 2, row, step, 4), word c & 3
 *       5 re-noise         (0, row, step, 5): word 0 token (entropy-bounded)
 *       6 self-cond drop   (0, b, step, 6): word 0 keep if < 2^31
 *     A word w becomes u = (2 (w >> 9) + 1) 2^-24 for a Gumbel variate
 *     -ln(-ln u), u = w 2^-32 for a comparison with a probability, and
 *     floor(w n / 2^32) for an index in [0, n).
 */
#ifndef DG_H_
#define DG_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef struct CUstream_st* dg_stream_t; /* same type as cudaStream_t */

typedef enum dg_status {
    DG_OK = 0,
    DG_ERR_INVALID_ARG = 1, /* a size, enum, pointer or scalar is out of range */
    DG_ERR_ALIGNMENT = 2,   /* a pointer or leading dimension breaks the 16-byte rule */
    DG_ERR_WORKSPACE = 3,   /* workspace missing or smaller than the size query */
    DG_ERR_CUDA = 4,        /* a CUDA runtime call failed (message has the CUDA error) */
    DG_ERR_UNSUPPORTED = 5  /* valid request the library does not handle (e.g. no sm_100 device) */
} dg_status;

typedef enum dg_dtype { DG_F32 = 0, DG_BF16 = 1 } dg_dtype;

/* Noise schedule kappa_t.  The pages fix only kappa_0 = 1, kappa_1 = 0 and
 * monotone decrease; the forms are: LINEAR 1 - t, COSINE cos^2(pi t / 2). */
typedef enum dg_schedule { DG_SCHED_LINEAR = 0, DG_SCHED_COSINE = 1 } dg_schedule;

/* How x0_hat is drawn from p0 = softmax(l * inv_tau).
 * SAMPLE: two-level Gumbel-max.  Level 1 scores each chunk of
 *   DG_GUMBEL_CHUNK consecutive ids (the last one ragged) with its
 *   log-sum-exp plus a chunk Gumbel variate; level 2 takes
 *   argmax_v l'_v + G_v inside the winning chunk.  Ties go to the lowest
 *   chunk, then the lowest id.  This draws exactly from softmax(l'); with
 *   V <= DG_GUMBEL_CHUNK it is plain Gumbel-max.
 * GREEDY: x0_hat = argmax_v l_v (lowest id on ties). */
typedef enum dg_x0_mode { DG_X0_SAMPLE = 0, DG_X0_GREEDY = 1 } dg_x0_mode;

#define DG_GUMBEL_CHUNK 512
#define DG_MAX_CANVASES 256 /* canvases (B, n_seq) per call */
#define DG_MAX_CANVAS_ROWS 1024 /* C for the per-canvas decisions (acceptance, stopping) */
#define DG_MAX_VOCAB (1 << 30) /* V for every call that reads logits rows (ids stay in 32 bits with headroom) */

/* Human-readable reason for the last failure on this thread ("" if none). */
const char* dg_last_error(void);
/* Library version string. */
const char* dg_version(void);
/* Number of kernels this library has launched in this process so far. */
uint64_t dg_launch_count(void);
/* Synchronizes the current device, then stores in *code (and clears) the
 * library's device error words (the largest code they hold): 0 if no kernel
 * has reported a problem, 1 if a kernel gave up on a bounded wait (its
 * outputs are then incomplete), 2 if a device-side check failed.  Every wait
 * inside the library's kernels is bounded (about two seconds), so a stalled
 * pipeline ends with code 1 instead of hanging the device.  Code 2 comes only
 * from the checks build of the library (libdg_checks.so, DG_CHECKS=1), whose
 * kernels verify the token ids and canvas indices they are given and their
 * own index invariants, and skip an access that would fail a check. */
int dg_device_error(int* code);

/* ------------------------------------------------------------------------ */
/* Sampler step (section "Method": p0 = Softmax(L_t / tau_t) and             */
/* x_{t-dt} ~ Step(x_t, p0)).  For each row r = b*C + i of B canvases:        */
/*   lse[r]      = log sum_v exp(l'_v),  l' = logits[r, :V] * inv_tau[b]     */
/*   max_prob[r] = max_v p0_v,  entropy[r] = -sum_v p0_v ln p0_v             */
/*   argmax[r]   = argmax_v logits[r, v] (lowest v on ties)                  */
/*   x0_hat[r]   ~ p0 (mode SAMPLE) or argmax[r] (mode GREEDY)               */
/*   x_next[r]   ~ P(X_s | X_t = x_t[r], X_0 = x0_hat[r]), s = max(t - dt, 0)*/
/*                 the exact posterior of the forward path; branch[r] = 0    */
/*                 stayed at x_t, 1 jumped to x0_hat, 2 drew a uniform token.*/
/*                 If kappa(s) <= kappa(t) (dt = 0) x_next = x_t, branch 0.  */
/* logits: device, DG_F32 or DG_BF16, [B*C, ld] (ld >= V).                   */
/* x_t: device int32 [B*C], ids in [0, V).                                   */
/* t, dt: host double [B], 0 <= t <= 1, dt >= 0.                             */
/* inv_tau: host float [B] (> 0, finite) or NULL for 1.                      */
/* Outputs (device, [B*C]): x_next int32 (required); x0_hat, argmax int32,   */
/* max_prob, lse, entropy float32, branch uint8 -- each may be NULL.         */
/* 1 <= B <= DG_MAX_CANVASES, C >= 1, 1 <= V <= DG_MAX_VOCAB, B*C < 2^31.   */
/* ------------------------------------------------------------------------ */
size_t dg_sampler_step_workspace_size(int32_t rows, int32_t V);

int dg_sampler_step(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t, int32_t B,
                    int32_t C, int32_t V, int schedule, const double* t, const double* dt,
                    const float* inv_tau, uint64_t seed, uint32_t step, int x0_mode,
                    int32_t* x_next, int32_t* x0_hat, int32_t* argmax, float* max_prob,
                    float* lse, float* entropy, uint8_t* branch, void* workspace,
                    size_t workspace_bytes, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Self-conditioning input (section "Method": z = FFW(p0 E)).  The trained   */
/* FFW is not part of this library; it computes the expected embedding      */
/*   z[r, :] = sum_v p0[r, v] E[v, :],  p0 = softmax(logits[r, :V] * inv_tau[b])*/
/* on the tensor cores (bf16 operands, fp32 accumulation), z stored bf16.    */
/* logits: device DG_F32 or DG_BF16 [B*C, ld].                              */
/* lse: device float [B*C] = log-sum-exp of logits*inv_tau per row, exactly  */
/*   as dg_sampler_step writes it; or NULL, in which case the library runs  */
/*   its own statistics pass first.                                          */
/* E: device [V, d] row-major, DG_BF16 (DG_F32 is rounded to bf16 into the   */
/*   workspace first).  d is a multiple of 64, 64 <= d <= 16384.             */
/* z: device bf16 [B*C, d] row-major.                                        */
/* ------------------------------------------------------------------------ */
size_t dg_selfcond_workspace_size(int32_t rows, int32_t V, int32_t d, int logits_dtype,
                                  int embed_dtype, int have_lse);

int dg_selfcond(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C, int32_t V,
                const float* inv_tau, const float* lse, const void* E, int embed_dtype, int32_t d,
                void* z, void* workspace, size_t workspace_bytes, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* One whole sampler step with its self-conditioning input (section         */
/* "Method": p0, z = p0 E and x_{t-dt} ~ Step(x_t, p0) of one iteration):    */
/* dg_sampler_step followed by dg_selfcond on the step's own lse, in one    */
/* call.  The contraction is launched as a programmatic dependent of the    */
/* logits pass, so its set-up and its copies of E and of the logits overlap */
/* the end of the pass; it reads lse only after the pass has completed.     */
/* Arguments: those of dg_sampler_step (lse required), then those of        */
/* dg_selfcond (E, embed_dtype, d, z and its own workspace, sized by         */
/* dg_selfcond_workspace_size(B*C, V, d, logits_dtype, embed_dtype, 1)).    */
/* All arguments are checked before anything is launched.                  */
/* ------------------------------------------------------------------------ */
int dg_sampler_selfcond_step(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t,
                             int32_t B, int32_t C, int32_t V, int schedule, const double* t,
                             const double* dt, const float* inv_tau, uint64_t seed, uint32_t step,
                             int x0_mode, int32_t* x_next, int32_t* x0_hat, int32_t* argmax,
                             float* max_prob, float* lse, float* entropy, uint8_t* branch,
                             void* workspace, size_t workspace_bytes, const void* E,
                             int embed_dtype, int32_t d, void* z, void* z_workspace,
                             size_t z_workspace_bytes, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Training-side forward corruption (section "Method": forward path, noisy   */
/* tokens drawn uniformly from the vocabulary; section "Dataset": P + K*C    */
/* layout, one loss canvas per sequence chosen uniformly).                   */
/* x0: device int32 [n_seq, P + K*C].  Prompt tokens are copied; each canvas*/
/* token j of sequence b is kept if w0 2^-32 < kappa(t[b]) and otherwise set*/
/* to floor(w1 V / 2^32).  canvas_idx[b] = floor(w0' K / 2^32).               */
/* t: host double [n_seq] in [0, 1].  x_t: device int32 like x0 (may not     */
/* alias x0).  canvas_idx: device int32 [n_seq] or NULL.  No workspace.      */
/* ------------------------------------------------------------------------ */
int dg_forward_noise(const int32_t* x0, int32_t n_seq, int32_t P, int32_t K, int32_t C, int32_t V,
                     int schedule, const double* t, uint64_t seed, int32_t* x_t,
                     int32_t* canvas_idx, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Canvas cross-entropy (section "Method": L = -sum_i log p(x_0^i | ...)) on */
/* the chosen canvas of each sequence (section "Dataset").                   */
/* logits: device DG_F32 or DG_BF16 [n_seq*C, ld]; row b*C + i predicts      */
/* target x0[b, P + canvas_idx[b]*C + i].  Outputs (device float):           */
/*   loss_rows [n_seq*C] = lse - logit[target], lse_rows [n_seq*C] (may be   */
/*   NULL), loss_seq [n_seq] = sum over the C rows (may be NULL).            */
/* canvas_idx: device int32 [n_seq], values in [0, K).                       */
/* ------------------------------------------------------------------------ */
size_t dg_canvas_ce_workspace_size(int32_t n_seq, int32_t C, int32_t V);

int dg_canvas_ce(const void* logits, int logits_dtype, int64_t ld, const int32_t* x0,
                 const int32_t* canvas_idx, int32_t n_seq, int32_t P, int32_t K, int32_t C,
                 int32_t V, float* loss_rows, float* loss_seq, float* lse_rows, void* workspace,
                 size_t workspace_bytes, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Temperature schedule (section "Method", sampler paragraph: tau_t < 1 is  */
/* annealed linearly over the denoising time scale from tau_max = 0.8 to    */
/* tau_min = 0.4).  Host only: inv_tau[b] = 1 / (tau_min + (tau_max -       */
/* tau_min) clamp(t[b], 0, 1)), ready for the inv_tau arguments above.      */
/* t: host double [B] (not NaN); inv_tau: host float [B].  tau_max, tau_min */
/* finite and > 0.  Returns DG_ERR_INVALID_ARG otherwise.                   */
/* ------------------------------------------------------------------------ */
int dg_tau_linear(const double* t, int32_t B, double tau_max, double tau_min, float* inv_tau);

/* ------------------------------------------------------------------------ */
/* Entropy-bounded acceptance (section "Method", sampler paragraph: tokens  */
/* are accepted in ascending order of entropy while an error bound stays    */
/* strictly below a tolerance; every other token is re-noised uniformly at  */
/* random).  Per canvas b of C rows r = b*C + i:                            */
/*   q_i = floor(clamp(entropy[r], 0, 64) 2^32)   (NaN counts as 64)        */
/*   order the rows by ascending (q_i, i); the k-th of that order is        */
/*   accepted iff q_(1) + ... + q_(k) < ceil(eps 2^32)                      */
/*   x_next[r] = accepted ? x0_hat[r] : floor(w0 V / 2^32),                 */
/*   w0 = Philox4x32-10(counter (0, r, step, 5), key seed) word 0.          */
/* The bound of an accepted set is read as the sum of its entropies (an     */
/* upper bound on its total correlation); the pages give no formula.        */
/* entropy: device float [B*C]; x0_hat: device int32 [B*C].                 */
/* Outputs (device): x_next int32 [B*C] (required), accepted uint8 [B*C]     */
/* and n_accepted int32 [B] (each may be NULL).  1 <= B <= DG_MAX_CANVASES, */
/* 1 <= C <= DG_MAX_CANVAS_ROWS (DG_ERR_UNSUPPORTED above), eps not NaN.    */
/* One CTA per canvas, no workspace.                                        */
/* ------------------------------------------------------------------------ */
int dg_entropy_accept(const float* entropy, const int32_t* x0_hat, int32_t B, int32_t C, int32_t V,
                      double eps, uint64_t seed, uint32_t step, int32_t* x_next, uint8_t* accepted,
                      int32_t* n_accepted, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Adaptive stopping (section "Method", sampler paragraph: stop when the    */
/* canvas-mean predicted entropy is below a threshold and the deterministic */
/* predictions of two consecutive steps are identical).  Per canvas b:      */
/*   stop[b] = sum_i q_i < ceil(theta C 2^32)  and  argmax == argmax_prev   */
/*             at every row of the canvas (q as in dg_entropy_accept);      */
/*   mean_entropy[b] = float((double) sum_i q_i 2^-32 / C).                 */
/* argmax, argmax_prev: device int32 [B*C]; argmax_prev NULL = no previous  */
/* step (stop is then 0).  Outputs device: stop uint8 [B], mean_entropy     */
/* float [B]; at least one non-NULL.  Limits as dg_entropy_accept.          */
/* ------------------------------------------------------------------------ */
int dg_adaptive_stop(const float* entropy, const int32_t* argmax, const int32_t* argmax_prev,
                     int32_t B, int32_t C, double theta, uint8_t* stop, float* mean_entropy,
                     dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Entropy-bounded sampler step: the statistics, argmax and x0_hat draw of  */
/* dg_sampler_step (its Step posterior is not applied), then the            */
/* acceptance and stopping decisions above on the step's own entropy and    */
/* argmax.  Two launches on `stream`.  Arguments as dg_sampler_step and the */
/* two functions above; x_next, x0_hat and entropy are required, argmax is  */
/* required when stop or mean_entropy is requested.  Workspace: the size   */
/* dg_sampler_step_workspace_size(B*C, V) gives, same contract.            */
/* ------------------------------------------------------------------------ */
int dg_sampler_step_eb(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C,
                       int32_t V, const float* inv_tau, uint64_t seed, uint32_t step, int x0_mode,
                       double eps, double theta, const int32_t* argmax_prev, int32_t* x_next,
                       int32_t* x0_hat, int32_t* argmax, float* max_prob, float* lse,
                       float* entropy, uint8_t* accepted, uint8_t* stop, float* mean_entropy,
                       void* workspace, size_t workspace_bytes, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Canvas cross-entropy backward (section "Method", loss equation): for row */
/* r = b*C + i with target y = x0[b, P + canvas_idx[b]*C + i],               */
/*   logits[r, v] <- g_seq[b] (exp(logits[r, v] - lse_rows[r]) - [v == y])  */
/* in place, rounded to bf16; rows whose target (or canvas index) is out of */
/* range become zero.  logits: device bf16 [n_seq*C, ld], V and ld multiples*/
/* of 8, 16-byte aligned.  lse_rows: device float [n_seq*C] as dg_canvas_ce */
/* writes it.  g_seq: device float [n_seq] (the upstream gradient of each   */
/* sequence's summed loss) or NULL for 1.  No workspace.                    */
/* ------------------------------------------------------------------------ */
int dg_canvas_ce_backward(void* logits, int64_t ld, const float* lse_rows, const int32_t* x0,
                          const int32_t* canvas_idx, int32_t n_seq, int32_t P, int32_t K,
                          int32_t C, int32_t V, const float* g_seq, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Self-conditioning drop for training (section "Dataset": for half of the  */
/* batch the decoder uses the previous pass's self-conditioning state, for  */
/* the other half that state is zero).  keep[b] = w0 < 2^31 with w0 from    */
/* Philox4x32-10(counter (0, b, step, 6), key seed); the C*d bf16 values of */
/* a dropped sequence are set to zero in place.  z: device bf16 [n_seq*C, d]*/
/* 16-byte aligned, C*d a multiple of 8.  keep: device uint8 [n_seq] or NULL.*/
/* ------------------------------------------------------------------------ */
int dg_selfcond_drop(void* z, int32_t n_seq, int32_t C, int32_t d, uint64_t seed, uint32_t step,
                     uint8_t* keep, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Feed-forward block on the self-conditioning input (section "Method":     */
/* z = FFW(p0 E), FFW a standard feed-forward network).  The pages name no  */
/* architecture; read as a two-layer perceptron without biases,            */
/*   hidden = gelu(z_in W1),  z_out = hidden W2,                            */
/* gelu in its tanh form.  Both layers run on the tensor cores (bf16        */
/* operands, fp32 accumulation); hidden and z_out are stored bf16.          */
/* z_in: device bf16 [rows, d]; W1: device bf16 [d, d_ff]; W2: device bf16  */
/* [d_ff, d]; hidden: device bf16 [rows, d_ff] (caller-owned scratch, also  */
/* an output); z_out: device bf16 [rows, d]; all row-major, 16-byte aligned */
/* and not aliased.  d, d_ff multiples of 64 in [64, 16384].  Workspace     */
/* (256-byte aligned, zeroed before first use like every workspace; it      */
/* holds the layers' fp32 split-K partial sums): dg_ffw_workspace_size      */
/* bytes (may be 0).  Up to four launches on `stream`: each layer's         */
/* contraction and its split sum, the second layer a programmatic           */
/* dependent of the first layer's last launch.                              */
/* ------------------------------------------------------------------------ */
size_t dg_ffw_workspace_size(int32_t rows, int32_t d, int32_t d_ff);

int dg_ffw(const void* z_in, int32_t rows, int32_t d, int32_t d_ff, const void* W1, const void* W2,
           void* hidden, void* z_out, void* workspace, size_t workspace_bytes, dg_stream_t stream);

/* ------------------------------------------------------------------------ */
/* Allocation-free sampler step.  The pages have no counterpart: this entry  */
/* point exists for callers that cannot allocate device memory where they   */
/* sample (a serving loop that must not call cudaMalloc, which can stall the */
/* whole device; a runtime that owns all device memory and passes the       */
/* library only input and output buffers).  It computes exactly what        */
/* dg_sampler_step computes, with the same arguments except the workspace: */
/* the scratch lives in a fixed device array of DG_NOALLOC_SCRATCH_BYTES     */
/* that every GPU loading the library holds until the process exits.        */
/*   - Limit: B*C rows of V ids must fit, i.e.                               */
/*     dg_sampler_step_workspace_size(B*C, V) <= DG_NOALLOC_SCRATCH_BYTES     */
/*     (256 rows of V = 262144 take about 2 MiB); larger requests return     */
/*     DG_ERR_WORKSPACE before anything is enqueued.                         */
/*   - The first call on a device looks up the array's device address       */
/*     (cudaGetSymbolAddress) with that device current; make that first call */
/*     before any stream capture on the device.                              */
/*   - Each call clears the part of the array it uses (an async memset on    */
/*     `stream`), so earlier contents never matter; all calls share the one  */
/*     array, so calls that overlap on the GPU race: serialise them (one     */
/*     stream, or events).  No call allocates or frees device memory.         */
/* ------------------------------------------------------------------------ */
#define DG_NOALLOC_SCRATCH_BYTES (4 * 1024 * 1024)

int dg_sampler_step_noalloc(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t,
                            int32_t B, int32_t C, int32_t V, int schedule, const double* t,
                            const double* dt, const float* inv_tau, uint64_t seed, uint32_t step,
                            int x0_mode, int32_t* x_next, int32_t* x0_hat, int32_t* argmax,
                            float* max_prob, float* lse, float* entropy, uint8_t* branch,
                            dg_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* DG_H_ */
