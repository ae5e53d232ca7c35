// Per-canvas sampler decisions and training-side elementwise passes.
//
// DiffusionGemma Technical Report (hyper.ai summary), section "Method", sampler paragraph:
//   tokens are accepted in ascending order of entropy while an error bound stays strictly below
//   a tolerance, the rest are re-noised uniformly at random; the sampler stops once the canvas-
//   mean entropy is below a threshold and two consecutive deterministic predictions agree.
// Same page, loss equation L = -sum_i log p(x0^i | x_t, z_t, H): its gradient with respect to
//   the logits, softmax - one-hot, written over the logits in place.
// Same page, section "Dataset": the self-conditioning state is used for half of the batch and
//   zero for the other half.
//
// canvas_decide_kernel: one CTA of kDecideThreads threads per canvas (C <= DG_MAX_CANVAS_ROWS), the
//   decisions of canvas_decide.cuh.  Launched as a programmatic dependent of the preceding kernel:
//   its CTAs may be placed while the logits pass's merge runs, and wait (griddepcontrol.wait) for
//   that grid's completion and its memory before reading any input.
// ce_backward_kernel: rows along grid y, 16-byte bf16 vectors of a row along grid x, in place.
// selfcond_drop_kernel: sequences along grid y; a fair Philox coin per sequence decides, dropped
//   rows are zeroed.
#include <algorithm>

#include "canvas_decide.cuh"
#include "common.cuh"
#include "kernels.cuh"

namespace dg {

namespace {

constexpr int kDecideThreads = 256;

__global__ void __launch_bounds__(kDecideThreads) canvas_decide_kernel(const __grid_constant__ DecideParams p) {
    __shared__ DecideShared sh;
    grid_dependency_wait();
    decide_canvas<kDecideThreads>(p, blockIdx.x, sh);
}

// grad = g_seq[b] (exp(l - lse) - [v == y]) over bf16 rows, in place.  Grid: x covers a row's
// 16-byte vectors (8 ids each), kCeVec per thread, consecutive threads on consecutive vectors;
// y strides over rows.
constexpr int kCeVec = 4;
__global__ void __launch_bounds__(256) ce_backward_kernel(const __grid_constant__ CeBackwardParams p) {
    const int32_t vec_per_row = p.V / 8;
    for (int32_t r = blockIdx.y; r < p.R; r += gridDim.y) {
        const int32_t b = r / p.C, i = r - b * p.C;
        const int32_t k = p.canvas_idx[b];
        int32_t y = -1;
        if (threadIdx.x == 0 && blockIdx.x == 0) DG_CHECK(g_ops_error, k >= 0 && k < p.K);  // caller's index
        if (k >= 0 && k < p.K) y = p.x0[static_cast<int64_t>(b) * p.seq_len + p.P + static_cast<int64_t>(k) * p.C + i];
        if (threadIdx.x == 0 && blockIdx.x == 0 && k >= 0 && k < p.K)
            DG_CHECK(g_ops_error, y >= 0 && y < p.V);  // a token id the caller gave
        uint4* row = reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(p.logits) + static_cast<int64_t>(r) * p.ld);
        const int32_t v_base = blockIdx.x * (kCeVec * 256) + threadIdx.x;
        if (y < 0 || y >= p.V) {
#pragma unroll
            for (int u = 0; u < kCeVec; ++u) {
                const int32_t vi = v_base + u * 256;
                if (vi < vec_per_row) row[vi] = make_uint4(0u, 0u, 0u, 0u);
            }
            continue;
        }
        const float g = p.g_seq ? p.g_seq[b] : 1.0f;
        const float nb = -p.lse[r] * kLog2e;
        uint4 in[kCeVec];
#pragma unroll
        for (int u = 0; u < kCeVec; ++u) {
            const int32_t vi = v_base + u * 256;
            in[u] = vi < vec_per_row ? row[vi] : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int u = 0; u < kCeVec; ++u) {
            const int32_t vi = v_base + u * 256;
            if (vi >= vec_per_row) continue;
            const uint32_t w[4] = {in[u].x, in[u].y, in[u].z, in[u].w};
            uint32_t o[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int32_t v = vi * 8 + 2 * j;
                float lo = g * ex2_approx(fmaf(bf16_lo(w[j]), kLog2e, nb));
                float hi = g * ex2_approx(fmaf(bf16_hi(w[j]), kLog2e, nb));
                if (v == y) lo -= g;
                if (v + 1 == y) hi -= g;
                o[j] = pack_bf16x2(lo, hi);
            }
            row[vi] = make_uint4(o[0], o[1], o[2], o[3]);
        }
    }
}

// Grid: y = sequence, x = 4 KB slices of its C*d values (256 threads x one 16-byte vector).
__global__ void __launch_bounds__(256) selfcond_drop_kernel(uint16_t* z, int64_t seq_elems, uint32_t key0,
                                                            uint32_t key1, uint32_t step, uint8_t* keep) {
    const int b = blockIdx.y;
    const uint4 w = philox4x32_10(make_uint4(0u, static_cast<uint32_t>(b), step, kDomScDrop), key0, key1);
    const bool kept = w.x < 0x80000000u;
    if (blockIdx.x == 0 && threadIdx.x == 0 && keep) keep[b] = static_cast<uint8_t>(kept);
    if (kept) return;
    uint4* dst = reinterpret_cast<uint4*>(z + static_cast<int64_t>(b) * seq_elems);
    const int64_t n = seq_elems / 8;
    for (int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; j < n;
         j += static_cast<int64_t>(gridDim.x) * blockDim.x)
        dst[j] = make_uint4(0u, 0u, 0u, 0u);
}

}  // namespace

cudaError_t read_and_clear_ops_error(int* out) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_ops_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_ops_error, &zero, sizeof(int));
    }
    *out = v;
    return e;
}

cudaError_t launch_canvas_decide(const DecideParams& p, int32_t B, cudaStream_t s) {
    if (B < 1 || p.C < 1 || p.C > DG_MAX_CANVAS_ROWS) return cudaErrorInvalidValue;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(B));
    cfg.blockDim = dim3(kDecideThreads);
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    const cudaError_t e = cudaLaunchKernelEx(&cfg, canvas_decide_kernel, p);
    if (e != cudaSuccess) return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_ce_backward(const CeBackwardParams& p, cudaStream_t s) {
    const int32_t vec_per_row = p.V / 8;
    const dim3 grid(static_cast<unsigned>((vec_per_row + kCeVec * 256 - 1) / (kCeVec * 256)),
                    static_cast<unsigned>(std::min<int32_t>(p.R, 65535)));
    ce_backward_kernel<<<grid, 256, 0, s>>>(p);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_selfcond_drop(uint16_t* z, int32_t n_seq, int64_t seq_elems, uint32_t key0, uint32_t key1,
                                 uint32_t step, uint8_t* keep, cudaStream_t s) {
    const int64_t n = seq_elems / 8;
    const dim3 grid(static_cast<unsigned>(std::min<int64_t>((n + 255) / 256, 1024)), static_cast<unsigned>(n_seq));
    selfcond_drop_kernel<<<grid, 256, 0, s>>>(z, seq_elems, key0, key1, step, keep);
    note_launches(1);
    return cudaGetLastError();
}

}  // namespace dg
