// Per-canvas sampler decisions (one CTA per canvas).
//
// DiffusionGemma Technical Report (hyper.ai summary), section "Method", sampler paragraph:
//   tokens are accepted in ascending order of entropy while an error bound stays strictly below a
//   tolerance, the rest are re-noised uniformly at random; the sampler stops once the canvas-mean
//   entropy is below a threshold and two consecutive deterministic predictions agree.
//
// Entropies become fixed-point integers q = floor(clamp(H, 0, 64) 2^32) (NaN -> 64), so sums and
// comparisons are exact and order-free.  Acceptance orders the canvas by the unique key
// (q << 10) | position: each warp sorts 32-key chunks with a register bitonic network, and a key's
// rank is its place in its own chunk plus, for every other chunk, the number of smaller keys found
// by a binary search of that chunk in shared memory.  The rank-ordered q are prefix-summed (a block
// scan) and the accepted set is the ranks whose prefix is below the tolerance.  Stopping: the sum of
// q against the threshold, and an all-equal test of the argmax canvas against the previous one.
// Per-row inputs may have been written by other CTAs of the same grid, so they are read through L2;
// every input is loaded once, up front, so the decisions wait on one round trip to memory.
#pragma once

#include "common.cuh"
#include "kernels.cuh"

namespace dg {

// Device error word of the per-canvas decisions and the other kernels of canvas_ops.cu (the one
// translation unit that includes this header): code 2 from a failed device-side check (checks
// library only).  Read and cleared by dg_device_error.
__device__ int g_ops_error = 0;

// Shared-memory scratch of one canvas's decisions (C up to DG_MAX_CANVAS_ROWS): the sorted 32-key
// chunks, the rank-ordered q, each position's rank, and the block reductions' slots.
static_assert(DG_MAX_CANVAS_ROWS <= 1024, "positions must fit the key's low 10 bits");
struct DecideSmall {
    long long warp_sum[32];
    int count[32];
};
struct DecideShared {
    unsigned long long chunks[DG_MAX_CANVAS_ROWS];
    long long sorted[DG_MAX_CANVAS_ROWS];
    int rank[DG_MAX_CANVAS_ROWS];
    DecideSmall small;
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

// Ascending bitonic sort of one key per lane across the warp (lane l ends with the l-th smallest).
__device__ __forceinline__ unsigned long long warp_sort32(unsigned long long key, int lane) {
#pragma unroll
    for (int k = 2; k <= 32; k <<= 1) {
#pragma unroll
        for (int j = k >> 1; j > 0; j >>= 1) {
            const unsigned long long other = __shfl_xor_sync(0xffffffffu, key, j);
            const bool keep_min = ((lane & j) == 0) == ((lane & k) == 0);
            key = keep_min ? (other < key ? other : key) : (other > key ? other : key);
        }
    }
    return key;
}

// Number of entries of the ascending 32-entry array a below key (a binary search of five halvings;
// the last test settles the one case, all 32 below, that the halvings leave open).
__device__ __forceinline__ int count_below32(const unsigned long long* a, unsigned long long key) {
    int pos = 0;
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) pos += (a[pos + s - 1] < key) ? s : 0;
    return pos + (a[pos] < key ? 1 : 0);
}

// The decisions of canvas b, by all kThreads threads of the CTA (C <= DG_MAX_CANVAS_ROWS).
// Warp w owns the 32-position chunks w, w + W, ... (W = kThreads / 32); lane l of a chunk loads
// position 32 * chunk + l, and positions past C get the key "infinity" (above every real key).
template <int kThreads>
__device__ void decide_canvas(const DecideParams& p, int b, DecideShared& sh) {
    constexpr int kWarps = kThreads / 32;
    constexpr int kChunksPerWarp = (DG_MAX_CANVAS_ROWS / 32 + kWarps - 1) / kWarps;
    constexpr int kPerThread = (DG_MAX_CANVAS_ROWS + kThreads - 1) / kThreads;
    constexpr unsigned long long kInf = ~0ull;
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int C = p.C;
    const int n_chunks = (C + 31) / 32;
    const int64_t r0 = static_cast<int64_t>(b) * C;
    const bool stopping = p.stop != nullptr || p.mean_entropy != nullptr;
    const bool compare = stopping && p.argmax_prev != nullptr;

    // ---- every input of this thread's positions, in one round trip
    unsigned long long key[kChunksPerWarp];
    int32_t x0[kChunksPerWarp];
    long long s = 0;
    int diff = 0;
#pragma unroll
    for (int u = 0; u < kChunksPerWarp; ++u) {
        const int i = (warp + u * kWarps) * 32 + lane;
        key[u] = kInf;
        x0[u] = 0;
        if (i < C) {
            const long long q = entropy_q(__ldcg(p.entropy + r0 + i));
            key[u] = (static_cast<unsigned long long>(q) << 10) | static_cast<unsigned>(i);
            s += q;
            if (p.x_next) x0[u] = __ldcg(p.x0_hat + r0 + i);
            if (compare) diff |= __ldcg(p.argmax + r0 + i) != __ldcg(p.argmax_prev + r0 + i);
        }
    }

    // ---- adaptive stopping: sum of q and the argmax comparison
    if (stopping) {
        const int any_diff = __syncthreads_or(diff);
        const long long total = block_inclusive_scan<kThreads>(s, sh.small.warp_sum);  // last thread: the sum
        if (tid == kThreads - 1) {
            const bool same = p.argmax_prev != nullptr && any_diff == 0;
            if (p.stop) p.stop[b] = static_cast<uint8_t>(total < p.stop_limit && same);
            if (p.mean_entropy)
                p.mean_entropy[b] = static_cast<float>(static_cast<double>(total) * (1.0 / 4294967296.0) /
                                                       static_cast<double>(C));
        }
    }
    if (!p.x_next) return;

    // ---- entropy-bounded acceptance: ranks by (q, position)
#pragma unroll
    for (int u = 0; u < kChunksPerWarp; ++u) {
        const int chunk = warp + u * kWarps;  // warp-uniform
        if (chunk < n_chunks) {
            key[u] = warp_sort32(key[u], lane);
            sh.chunks[chunk * 32 + lane] = key[u];
        }
    }
    __syncthreads();
#pragma unroll
    for (int u = 0; u < kChunksPerWarp; ++u) {
        const int chunk = warp + u * kWarps;
        if (chunk < n_chunks && key[u] != kInf) {
            int r = 0;  // the own chunk contributes the key's lane: keys are unique
#pragma unroll 4
            for (int c = 0; c < n_chunks; ++c) r += count_below32(sh.chunks + c * 32, key[u]);
            if (DG_CHECKED(g_ops_error, r < C && static_cast<int>(key[u] & 1023u) < C)) {
                sh.sorted[r] = static_cast<long long>(key[u] >> 10);
                sh.rank[key[u] & 1023u] = r;
            }
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
    const long long incl = block_inclusive_scan<kThreads>(run, sh.small.warp_sum);
    const long long base = incl - run;
    int cnt = 0;
#pragma unroll
    for (int u = 0; u < kPerThread; ++u) {
        const int k = tid * kPerThread + u;
        cnt += (k < C) & (base + local[u] < p.accept_limit);
    }
    // the accepted ranks are a prefix (q >= 0): their number is the count of passing prefixes
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if (lane == 0) sh.small.count[warp] = cnt;
    __syncthreads();
    int n_acc = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) n_acc += sh.small.count[w];
    if (tid == 0 && p.n_accepted) p.n_accepted[b] = n_acc;
#pragma unroll
    for (int u = 0; u < kChunksPerWarp; ++u) {
        const int i = (warp + u * kWarps) * 32 + lane;
        if (i < C) {
            const int64_t r = r0 + i;
            const bool acc = sh.rank[i] < n_acc;
            int32_t x = x0[u];
            if (acc) DG_CHECK(g_ops_error, x >= 0 && x < p.V);  // an x0_hat the caller gave
            if (!acc) {
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
