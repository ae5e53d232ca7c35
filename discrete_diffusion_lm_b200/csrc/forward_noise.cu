// Training-side forward corruption.
//
// DiffusionGemma Technical Report (hyper.ai summary), section "Method": the forward path
// kappa_t delta(x_t, x_0) + (1 - kappa_t)/V factorises over token coordinates, and the corruption
// draws noisy tokens uniformly from the vocabulary.  Section "Dataset": a training sequence is P
// prompt tokens followed by K canvases of C tokens; the decoder loss uses one canvas per sequence,
// chosen uniformly.
//
// One thread per token.  Prompt tokens are copied.  Canvas token j of sequence b takes Philox
// counter (j, b, 0, 2): it is kept when word 0 is below the sequence's threshold ceil(kappa_b 2^32)
// and otherwise replaced by floor(word1 V / 2^32).  Thread 0 of each sequence also draws the loss
// canvas floor(w K / 2^32) from counter (0, b, 0, 3).  The whole call is a few tens of KB, so it is
// bounded by launch latency, not by memory.
#include "common.cuh"
#include "kernels.cuh"

namespace dg {

namespace {

// Device error word of this file's kernel: code 2 from a failed device-side check (checks library
// only).  Read and cleared by dg_device_error.
__device__ int g_noise_error = 0;

constexpr int kNoiseThreads = 256;

__global__ void __launch_bounds__(kNoiseThreads) forward_noise_kernel(const __grid_constant__ NoiseParams p) {
    const int32_t b = blockIdx.y;
    const int64_t j = static_cast<int64_t>(blockIdx.x) * kNoiseThreads + threadIdx.x;
    if (j == 0 && p.canvas_idx) {
        const uint4 w = philox4x32_10(make_uint4(0u, static_cast<uint32_t>(b), 0u, kDomCanvas), p.key0, p.key1);
        p.canvas_idx[b] = word_to_index(w.x, p.K);
    }
    if (j >= p.seq_len) return;
    const int64_t at = static_cast<int64_t>(b) * p.seq_len + j;
    int32_t tok = p.x0[at];
    DG_CHECK(g_noise_error, tok >= 0 && tok < p.V);  // a token id the caller gave
    if (j >= p.P) {
        const uint4 w = philox4x32_10(make_uint4(static_cast<uint32_t>(j), static_cast<uint32_t>(b), 0u, kDomNoise),
                                      p.key0, p.key1);
        if (!(static_cast<unsigned long long>(w.x) < p.keep_thr[b])) tok = word_to_index(w.y, p.V);
    }
    p.x_t[at] = tok;
}

}  // namespace

cudaError_t read_and_clear_noise_error(int* out) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_noise_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_noise_error, &zero, sizeof(int));
    }
    *out = v;
    return e;
}

cudaError_t launch_forward_noise(const NoiseParams& p, cudaStream_t s) {
    const long long bx = (p.seq_len + kNoiseThreads - 1) / kNoiseThreads;
    if (bx <= 0 || bx > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    forward_noise_kernel<<<dim3(static_cast<unsigned>(bx), p.n_seq), kNoiseThreads, 0, s>>>(p);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace dg
