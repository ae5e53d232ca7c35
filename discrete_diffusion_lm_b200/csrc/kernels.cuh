// Kernel parameter blocks and host-side launchers (internal to libdg).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dg.h"

namespace dg {

constexpr int kChunk = DG_GUMBEL_CHUNK;  // ids per level-1 Gumbel chunk

// Which epilogue the logits pass runs after the per-row merge.
enum PassKind : int {
    kPassSampler = 0,  // statistics + argmax + x0 draw + Step
    kPassStats = 1,    // log-sum-exp only (self-conditioning prepass)
    kPassCE = 2,       // cross-entropy against a target id + per-sequence sum
};

struct PassParams {
    const void* logits;
    int64_t ld;  // elements
    int32_t R, C, V;
    int32_t n_chunks;        // ceil(V / kChunk)
    int32_t groups_per_cta;  // 4-chunk groups per CTA, a multiple of the warps per CTA
    int32_t segs;            // CTAs per row
    unsigned long long* rec;  // [R, n_chunks, kRecWords] tagged record words (raw max, S, T), see logits_pass.cu
    unsigned* epoch;          // [2] call counter (tags the records) and the merge CTAs' ticket
    long long merge_wait_limit;  // cycles a merge waits for its row (0: the library default)
    // sampler
    const int32_t* x_t;
    uint32_t key0, key1, step;
    int32_t mode;
    int32_t* x_next;
    int32_t* x0_hat;
    int32_t* argmax;
    float* max_prob;
    float* lse;
    float* entropy;
    uint8_t* branch;
    // cross-entropy
    const int32_t* x0;
    const int32_t* canvas_idx;
    int32_t P, K;
    int64_t seq_len;
    float* loss_rows;
    float* loss_seq;
    uint32_t* seq_ticket;  // [n_seq], zero between calls
    // per canvas (sampler) -- Step thresholds on the 32-bit branch word, in [0, 2^32]
    float inv_tau[DG_MAX_CANVASES];
    unsigned long long thr_stay_diff[DG_MAX_CANVASES];  // x0_hat != x_t: stay if w0 < this
    unsigned long long thr_jump_diff[DG_MAX_CANVASES];  //               jump if w0 < this
    unsigned long long thr_stay_same[DG_MAX_CANVASES];  // x0_hat == x_t: stay if w0 < this
};

constexpr int kPassThreads = 128;
constexpr int kPassWarps = kPassThreads / 32;
constexpr int kRecWords = 3;  // 64-bit words per chunk record (bf16 logits use the first two)

cudaError_t launch_logits_pass(const PassParams& p, int kind, int is_bf16, cudaStream_t s);
// Test hook: the statistics merge kernel alone, with nothing counting the rows (its waits expire).
cudaError_t launch_merge_only(const PassParams& p, int is_bf16, cudaStream_t s);
// Reads and clears the logits pass's device error word (1 = a merge's bounded wait expired).
cudaError_t read_and_clear_pass_error(int* out);

struct NoiseParams {
    const int32_t* x0;
    int32_t* x_t;
    int32_t* canvas_idx;
    int32_t n_seq, P, K, C, V;
    int64_t seq_len;
    uint32_t key0, key1;
    unsigned long long keep_thr[DG_MAX_CANVASES];  // keep if w0 < this, in [0, 2^32]
};

cudaError_t launch_forward_noise(const NoiseParams& p, cudaStream_t s);

// Self-conditioning contraction z = softmax(l') E on tcgen05 tensor cores.
struct SelfcondParams {
    const void* logits;  // [R, ld]
    int64_t ld;
    int32_t logits_bf16;
    const float* lse;    // [R]
    const uint16_t* E;   // bf16 [V, d]
    uint16_t* z;         // bf16 [R, d]
    float* partial;      // fp32 [splits, R, d] (when the vocabulary is split)
    int32_t R, C, V, d;
    long long wait_limit;  // cycles before a stalled wait aborts the CTA (0: the library default)
    int32_t fault_block;   // test hook: never issue the E copy of this 64-id block (-1: none)
    int32_t plain_a;       // 1: `logits` is a plain bf16 A operand [R, V] (no softmax, lse unused)
    int32_t act;           // epilogue activation on z: 0 none, 1 GELU (tanh form)
    int32_t dependent;     // 1: launch as a programmatic dependent of the preceding logits pass
    float inv_tau[DG_MAX_CANVASES];
};

size_t selfcond_partial_bytes(int32_t R, int32_t V, int32_t d, bool logits_bf16, bool plain_a = false);
cudaError_t launch_selfcond(const SelfcondParams& p, cudaStream_t s);
cudaError_t launch_convert_f32_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t s);
// One thread waits on a barrier nothing arrives on; the bounded wait must give up (test).
cudaError_t launch_bounded_wait_test(long long limit_cycles, cudaStream_t s);
// Reads (synchronously) and clears the error word set by a kernel whose bounded wait expired.
cudaError_t read_and_clear_device_error(int* out);
// The same for the error words of canvas_ops.cu and forward_noise.cu (device-side checks).
cudaError_t read_and_clear_ops_error(int* out);
cudaError_t read_and_clear_noise_error(int* out);

// Per-canvas sampler decisions: entropy-bounded acceptance with uniform re-noising, and the
// adaptive-stopping flag.  One CTA per canvas.  Null outputs skip their part (x_next == nullptr:
// no acceptance; stop and mean_entropy both nullptr: no stopping test).
struct DecideParams {
    const float* entropy;        // [B*C]
    const int32_t* x0_hat;       // [B*C]           (acceptance)
    const int32_t* argmax;       // [B*C]           (stopping)
    const int32_t* argmax_prev;  // [B*C] or null   (stopping; null: no previous step)
    int32_t C, V;
    long long accept_limit;      // accept while the rank-ordered prefix sum of q is below this
    long long stop_limit;        // stop needs sum q below this
    uint32_t key0, key1, step;
    int32_t* x_next;             // [B*C]
    uint8_t* accepted;           // [B*C] or null
    int32_t* n_accepted;         // [B] or null
    uint8_t* stop;               // [B] or null
    float* mean_entropy;         // [B] or null
};
cudaError_t launch_canvas_decide(const DecideParams& p, int32_t B, cudaStream_t s);

// Canvas cross-entropy gradient, in place over bf16 logits rows.
struct CeBackwardParams {
    void* logits;  // bf16 [R, ld], overwritten by the gradient
    int64_t ld;
    const float* lse;         // [R] saved by the forward pass
    const int32_t* x0;        // [n_seq, seq_len]
    const int32_t* canvas_idx;  // [n_seq]
    const float* g_seq;       // [n_seq] upstream gradient of each sequence's summed loss, or null (1)
    int32_t R, C, V, P, K;
    int64_t seq_len;
};
cudaError_t launch_ce_backward(const CeBackwardParams& p, cudaStream_t s);

// Zero the self-conditioning rows (C*d bf16 values per sequence) of sequences whose coin drops them.
cudaError_t launch_selfcond_drop(uint16_t* z, int32_t n_seq, int64_t seq_elems, uint32_t key0, uint32_t key1,
                                 uint32_t step, uint8_t* keep, cudaStream_t s);

// The sampler step behind the two C entry points (dg_sampler_step, dg_sampler_step_noalloc): all
// arguments are checked first; with clear_ws the workspace is then zeroed on the stream before the
// launches.  Returns a DG_* status.
int sampler_step_impl(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t, int32_t B, int32_t C,
                      int32_t V, int schedule, const double* t, const double* dt, const float* inv_tau, uint64_t seed,
                      uint32_t step, int x0_mode, int32_t* x_next, int32_t* x0_hat, int32_t* argmax, float* max_prob,
                      float* lse, float* entropy, uint8_t* branch, void* workspace, size_t workspace_bytes,
                      dg_stream_t stream, bool clear_ws);

// Multiprocessor count of the current device (cached per device).
int num_sms();

// Count of kernels launched by the library (for the launch-count query).
void note_launches(uint64_t n);

}  // namespace dg
