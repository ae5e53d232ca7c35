// Per-canvas sampler decisions, shared by the standalone decision kernel and the logits pass's
// merge kernel (which runs them for a canvas once the canvas's last row is merged).
//
// DiffusionGemma Technical Report (hyper.ai summary), section "Method", sampler paragraph:
//   tokens are accepted in ascending order of entropy while an error bound stays strictly below a
//   tolerance, the rest are re-noised uniformly at random; the sampler stops once the canvas-mean
//   entropy is below a threshold and two consecutive deterministic predictions agree.
//
// Entropies become fixed-point integers q = floor(clamp(H, 0, 64) 2^32) (NaN -> 64), so sums and
// comparisons are exact and order-free.  Acceptance: ranks by (q, position) are computed by
// counting in shared memory, the rank-ordered q are prefix-summed (a block scan) and the accepted
// set is the ranks whose prefix is below the tolerance.  Stopping: the sum of q against the
// threshold, and an all-equal test of the argmax canvas against the previous one.  Per-row inputs
// may have been written by other CTAs of the same grid, so they are read through L2.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace dg {

struct DecideShared {
    long long q[DG_MAX_CANVAS_ROWS];
    long long sorted[DG_MAX_CANVAS_ROWS];
    long long warp_sum[32];
    int count[32];
    int same;
};

__device__ __forceinline__ long long entropy_q(float h) {
    float x = h;
    if (!(x >= 0.f)) x = isnan(x) ? 64.f : 0.f;
    x = fminf(x, 64.f);
    return __float2ll_rd(x * 4294967296.f);  // exact: a power-of-two scale of a float
}

// Inclusive block-wide prefix sum of one 64-bit value per thread (kThreads threads).
template <int kThreads>
__device__ __forceinline__ long long block_inclusive_scan(long long v, long long* sh_warp) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const long long n = __shfl_up_sync(0xffffffffu, v, o);
        if (lane >= o) v += n;
    }
    if (lane == 31) sh_warp[warp] = v;
    __syncthreads();
    long long base = 0;
    for (int w = 0; w < warp; ++w) base += sh_warp[w];
    __syncthreads();
    return v + base;
}

// The decisions of canvas b, by all kThreads threads of the CTA (C <= DG_MAX_CANVAS_ROWS).
template <int kThreads>
__device__ void decide_canvas(const DecideParams& p, int b, DecideShared& sh) {
    constexpr int kPerThread = (DG_MAX_CANVAS_ROWS + kThreads - 1) / kThreads;
    const int tid = threadIdx.x;
    const int C = p.C;
    const int64_t r0 = static_cast<int64_t>(b) * C;
    if (tid == 0) sh.same = 1;
    for (int i = tid; i < C; i += kThreads) sh.q[i] = entropy_q(__ldcg(p.entropy + r0 + i));
    __syncthreads();

    // ---- adaptive stopping: sum of q and the argmax comparison
    if (p.stop || p.mean_entropy) {
        long long s = 0;
        int diff = 0;
        for (int i = tid; i < C; i += kThreads) {
            s += sh.q[i];
            if (p.argmax_prev && __ldcg(p.argmax + r0 + i) != __ldcg(p.argmax_prev + r0 + i)) diff = 1;
        }
        if (__any_sync(0xffffffffu, diff) && (tid & 31) == 0) sh.same = 0;
        const long long total = block_inclusive_scan<kThreads>(s, sh.warp_sum);  // last thread: the sum
        if (tid == kThreads - 1) {
            const bool same = p.argmax_prev != nullptr && sh.same != 0;
            if (p.stop) p.stop[b] = static_cast<uint8_t>(total < p.stop_limit && same);
            if (p.mean_entropy)
                p.mean_entropy[b] = static_cast<float>(static_cast<double>(total) * (1.0 / 4294967296.0) /
                                                       static_cast<double>(C));
        }
    }
    if (!p.x_next) return;

    // ---- entropy-bounded acceptance
    int rank[kPerThread];
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int i = tid + u * kThreads;
        rank[u] = 0;
        if (i < C) {
            const long long qi = sh.q[i];
            int r = 0;
            for (int j = 0; j < C; ++j) {
                const long long qj = sh.q[j];
                r += (qj < qi) | ((qj == qi) & (j < i));
            }
            rank[u] = r;
            sh.sorted[r] = qi;
        }
    }
    __syncthreads();
    // thread t scans ranks kPerThread t .. kPerThread t + kPerThread - 1
    long long local[kPerThread];
    long long run = 0;
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int k = tid * kPerThread + u;
        run += k < C ? sh.sorted[k] : 0;
        local[u] = run;
    }
    const long long incl = block_inclusive_scan<kThreads>(run, sh.warp_sum);
    const long long base = incl - run;
    int cnt = 0;
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int k = tid * kPerThread + u;
        cnt += (k < C) & (base + local[u] < p.accept_limit);
    }
    // the accepted ranks are a prefix (q >= 0): their number is the count of passing prefixes
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if ((tid & 31) == 0) sh.count[tid >> 5] = cnt;
    __syncthreads();
    int n_acc = 0;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) n_acc += sh.count[w];
    if (tid == 0 && p.n_accepted) p.n_accepted[b] = n_acc;
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int i = tid + u * kThreads;
        if (i < C) {
            const int64_t r = r0 + i;
            const bool acc = rank[u] < n_acc;
            int32_t x;
            if (acc) {
                x = __ldcg(p.x0_hat + r);
            } else {
                const uint4 w =
                    philox4x32_10(make_uint4(0u, static_cast<uint32_t>(r), p.step, kDomRenoise), p.key0, p.key1);
                x = word_to_index(w.x, p.V);
            }
            p.x_next[r] = x;
            if (p.accepted) p.accepted[r] = static_cast<uint8_t>(acc);
        }
    }
}

}  // namespace dg
