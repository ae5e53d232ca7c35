// Device helpers shared by the sampler kernels (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/dg.h"

namespace dg {

constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kNegBig = -1.0e30f;  // -inf logits are clamped here before any arithmetic

// Device-side checks, compiled in by the checks library (DG_CHECKS=1) and away otherwise.
//   DG_CHECK(word, cond)    statement: when cond fails, code 2 goes to the device error word;
//   DG_CHECKED(word, cond)  expression guarding an access: the same, and false skips the access.
// In the normal build cond is not evaluated: DG_CHECK is a no-op and DG_CHECKED is true.
#if defined(DG_CHECKS) && DG_CHECKS
#define DG_CHECK(word, cond)          \
    do {                              \
        if (!(cond)) atomicMax(&(word), 2); \
    } while (0)
#define DG_CHECKED(word, cond) ((cond) ? true : (atomicMax(&(word), 2), false))
#else
#define DG_CHECK(word, cond) ((void)0)
#define DG_CHECKED(word, cond) true
#endif

// ---------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon, Moraes, Dror, Shaw, "Parallel random numbers: as easy as 1, 2, 3",
// SC'11): ten rounds; each multiplies counter words 0 and 2 by the two published multipliers,
// xors the high halves into the other words together with the key, and bumps the key by the
// published Weyl constants between rounds.
// ---------------------------------------------------------------------------------------------
constexpr uint32_t kPhiloxMulA = 0xD2511F53u;
constexpr uint32_t kPhiloxMulB = 0xCD9E8D57u;
constexpr uint32_t kPhiloxWeylA = 0x9E3779B9u;
constexpr uint32_t kPhiloxWeylB = 0xBB67AE85u;

enum : uint32_t {
    kDomTokenGumbel = 0,
    kDomStep = 1,
    kDomNoise = 2,
    kDomCanvas = 3,
    kDomChunkGumbel = 4,
    kDomRenoise = 5,  // entropy-bounded sampler: the re-noised token of a rejected position
    kDomScDrop = 6,   // training: the self-conditioning keep/drop coin of a sequence
};

__device__ __forceinline__ uint4 philox4x32_10(uint4 c, uint32_t k0, uint32_t k1) {
#pragma unroll
    for (int round = 0; round < 10; ++round) {
        if (round > 0) {
            k0 += kPhiloxWeylA;
            k1 += kPhiloxWeylB;
        }
        const uint32_t hi_a = __umulhi(kPhiloxMulA, c.x), lo_a = kPhiloxMulA * c.x;
        const uint32_t hi_b = __umulhi(kPhiloxMulB, c.z), lo_b = kPhiloxMulB * c.z;
        c = make_uint4(hi_b ^ c.y ^ k0, lo_b, hi_a ^ c.w ^ k1, lo_a);
    }
    return c;
}

__device__ __forceinline__ uint32_t word_of(const uint4& w, uint32_t i) {
    return i == 0 ? w.x : i == 1 ? w.y : i == 2 ? w.z : w.w;
}

// Gumbel variate -ln(-ln u) with u = (2 (w >> 9) + 1) 2^-24, exact in fp32.  Full-precision
// logf: near u -> 1 the inner log is tiny and its relative accuracy sets the variate's.
__device__ __forceinline__ float gumbel_from_word(uint32_t w) {
    const float u = static_cast<float>(2u * (w >> 9) + 1u) * 0x1p-24f;
    return -logf(-logf(u));
}

// floor(w n / 2^32)
__device__ __forceinline__ int32_t word_to_index(uint32_t w, int32_t n) {
    return static_cast<int32_t>(__umulhi(w, static_cast<uint32_t>(n)));
}

// ---------------------------------------------------------------------------------------------
// Memory helpers.
// ---------------------------------------------------------------------------------------------
// Streaming 16-byte load: read-only path, no L1 allocation (each byte is read once).
__device__ __forceinline__ uint4 ld_stream_v4(const void* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// L2-coherent loads for data written by other CTAs of the same launch.
__device__ __forceinline__ float4 ld_cg_f4(const float4* p) { return __ldcg(p); }
__device__ __forceinline__ float ld_cg_f(const float* p) { return __ldcg(p); }

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// Two floats rounded to nearest-even bf16, packed low/high.
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    const __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<const uint32_t*>(&h);
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

__device__ __forceinline__ float load_logit(const void* row, int32_t v, int is_bf16) {
    if (is_bf16) {
        const uint16_t h = reinterpret_cast<const uint16_t*>(row)[v];
        return __uint_as_float(static_cast<uint32_t>(h) << 16);
    }
    return reinterpret_cast<const float*>(row)[v];
}

// ---------------------------------------------------------------------------------------------
// Shared-memory barriers (mbarrier).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes)
                 : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}
// Makes barrier initialisation visible to the other threads and to the copy engine.
__device__ __forceinline__ void fence_barrier_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

// ---------------------------------------------------------------------------------------------
// Programmatic dependent launch.  A kernel launched with programmatic stream serialization may
// start while its predecessor in the stream still runs; before it reads anything the
// predecessor writes it waits for the predecessor's completion (and memory).  A kernel lets its
// dependents start early by triggering; both are no-ops without such a dependency.
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ void grid_dependency_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// Warp / block reductions (blockDim.x == 32 * kWarpsPerBlock, all threads participate).
// ---------------------------------------------------------------------------------------------
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}
__device__ __forceinline__ int warp_min_int(int v) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
// (value, index): larger value wins, equal values go to the smaller index.
__device__ __forceinline__ void warp_argmax(float& v, int& i) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, v, o);
        const int oi = __shfl_xor_sync(0xffffffffu, i, o);
        if (ov > v || (ov == v && oi < i)) {
            v = ov;
            i = oi;
        }
    }
}

template <int kWarps>
__device__ __forceinline__ float block_max(float v, float* sh) {
    v = warp_max(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) sh[w] = v;
    __syncthreads();
    v = l < kWarps ? sh[l] : -INFINITY;
    return warp_max(v);
}
template <int kWarps>
__device__ __forceinline__ float block_sum(float v, float* sh) {
    v = warp_sum(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) sh[w] = v;
    __syncthreads();
    v = l < kWarps ? sh[l] : 0.f;
    return warp_sum(v);
}
template <int kWarps>
__device__ __forceinline__ int block_min_int(int v, int* sh) {
    v = warp_min_int(v);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) sh[w] = v;
    __syncthreads();
    v = l < kWarps ? sh[l] : 0x7fffffff;
    return warp_min_int(v);
}
template <int kWarps>
__device__ __forceinline__ void block_argmax(float& v, int& i, float* shv, int* shi) {
    warp_argmax(v, i);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) {
        shv[w] = v;
        shi[w] = i;
    }
    __syncthreads();
    v = l < kWarps ? shv[l] : -INFINITY;
    i = l < kWarps ? shi[l] : 0x7fffffff;
    warp_argmax(v, i);
}
// Two independent (value, index) argmax reductions in one exchange; shv and shi hold 2 kWarps.
template <int kWarps>
__device__ __forceinline__ void block_argmax2(float& v0, int& i0, float& v1, int& i1, float* shv, int* shi) {
    warp_argmax(v0, i0);
    warp_argmax(v1, i1);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) {
        shv[w] = v0;
        shi[w] = i0;
        shv[kWarps + w] = v1;
        shi[kWarps + w] = i1;
    }
    __syncthreads();
    v0 = l < kWarps ? shv[l] : -INFINITY;
    i0 = l < kWarps ? shi[l] : 0x7fffffff;
    v1 = l < kWarps ? shv[kWarps + l] : -INFINITY;
    i1 = l < kWarps ? shi[kWarps + l] : 0x7fffffff;
    warp_argmax(v0, i0);
    warp_argmax(v1, i1);
}
// Two sums in one exchange; sh holds 2 kWarps.
template <int kWarps>
__device__ __forceinline__ void block_sum2(float& a, float& b, float* sh) {
    a = warp_sum(a);
    b = warp_sum(b);
    const int w = threadIdx.x >> 5, l = threadIdx.x & 31;
    __syncthreads();
    if (l == 0) {
        sh[w] = a;
        sh[kWarps + w] = b;
    }
    __syncthreads();
    a = warp_sum(l < kWarps ? sh[l] : 0.f);
    b = warp_sum(l < kWarps ? sh[kWarps + l] : 0.f);
}

}  // namespace dg
