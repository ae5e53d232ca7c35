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
    float4* rec;             // [R, n_chunks] per-chunk (raw max, S, T, -)
    uint32_t* row_ticket;    // [R], zero between calls
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

cudaError_t launch_logits_pass(const PassParams& p, int kind, int is_bf16, cudaStream_t s);

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
    int32_t fault_block;   // test hook: never issue the E copy of this 32-id block (-1: none)
    float inv_tau[DG_MAX_CANVASES];
};

size_t selfcond_partial_bytes(int32_t R, int32_t V, int32_t d, bool logits_bf16);
cudaError_t launch_selfcond(const SelfcondParams& p, cudaStream_t s);
cudaError_t launch_convert_f32_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t s);
// One thread waits on a barrier nothing arrives on; the bounded wait must give up (test).
cudaError_t launch_bounded_wait_test(long long limit_cycles, cudaStream_t s);
// Reads (synchronously) and clears the error word set by a kernel whose bounded wait expired.
cudaError_t read_and_clear_device_error(int* out);

// Count of kernels launched by the library (for the launch-count query).
void note_launches(uint64_t n);

}  // namespace dg
