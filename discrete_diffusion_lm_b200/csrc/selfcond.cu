// Self-conditioning contraction z = softmax(l * inv_tau) E on the sm_100a tensor cores.
//
// DiffusionGemma Technical Report (hyper.ai summary), section "Method": the update
// z_{t-dt} = FFW(p0 E) with p0 = Softmax(L_t / tau_t) and E the token-embedding matrix.  The
// expected embedding p0 E is the dense contraction computed here (the trained FFW is not).
//
// One CTA computes a 128-row x kNT-column tile of z over a contiguous range of the vocabulary
// (split-K).  Per stage of kKBlock = 64 ids:
//   * a producer thread TMA-loads the E tile [64 ids x kNT] (MN-major, 128-byte swizzle, boxes of
//     64 columns) and the logits tile [128 rows x 64 ids] (128-byte swizzle);
//   * four softmax warps turn each thread's logits row into p = exp2(l * a - lse * log2 e), i.e.
//     softmax(l') with the row's log-sum-exp from the logits pass, round it to bf16 and write it
//     back in the K-major 128-byte-swizzled layout the tensor core reads as operand A;
//   * one thread issues tcgen05.mma (kind::f16, bf16 x bf16 -> fp32) into a TMEM accumulator of
//     128 lanes x kNT columns and commits the stage back to the producer.
// Because lse is known, p is final when it is formed: no running-max rescale of the accumulator is
// needed.  After the last stage the softmax warps read the accumulator out of TMEM (tcgen05.ld)
// and store bf16 z, or fp32 partial sums that a second kernel adds in a fixed order.
// Every mbarrier wait is bounded: on expiry the CTA records an error, stops issuing work, waits
// (bounded) for its in-flight copies and frees its TMEM.
#include <cuda.h>  // CUtensorMap and its enums (the encoder itself is fetched from the driver at run time)

#include <algorithm>
#include <atomic>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "kernels.cuh"

namespace dg {

__device__ int g_device_error = 0;  // set by a kernel whose bounded wait expired

namespace {

constexpr int kKBlock = 64;  // vocabulary ids per pipeline stage
constexpr int kTileM = 128;  // rows per CTA = TMEM lanes
constexpr int kNumSoftmaxWarps = 8;  // two groups of four; group g converts the stages i with i % 2 == g
constexpr int kGroupThreads = 128;
constexpr int kThreads = 64 + 32 * kNumSoftmaxWarps;  // producer warp, MMA warp, softmax warps
constexpr long long kWaitLimitCycles = 4000000000LL;  // about 2 s at the boost clock

struct alignas(64) KernelParams {
    CUtensorMap tm_logits;  // [R, V], box 128 rows x (64 bytes of ids)
    CUtensorMap tm_E;       // [V, d], box kKBlock ids x 64 columns
    CUtensorMap tm_out;     // pair kernel's TMA stores: z [R, d] bf16 (box 64 x 128) when splits == 1,
                            // else the partial sums [splits, R, d] fp32 (box 32 x 128 x 1)
    const float* lse;
    uint16_t* z;
    float* partial;
    int32_t R, C, V, d;
    int32_t n_tiles, splits, total_kb;
    long long wait_limit;  // cycles a wait may last before the CTA aborts
    int32_t fault_block;   // test hook: the E copy of this kKBlock-id block is never issued (-1: none)
    int32_t plain;         // 1: the A tiles are the bf16 operand as loaded (no softmax; lse unused)
    int32_t act;           // epilogue activation: 0 none, 1 GELU (tanh form)
    float inv_tau[DG_MAX_CANVASES];
};

// GELU, tanh form (Hendrycks and Gimpel, "Gaussian Error Linear Units", 2016), with the hardware
// tanh approximation (tanh.approx.f32, relative error about 2^-11, below the bf16 rounding of the
// result).
__device__ __forceinline__ float tanh_approx(float x) {
    float y;
    asm("tanh.approx.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float gelu_tanh(float x) {
    const float k0 = 0.7978845608028654f;  // sqrt(2 / pi)
    const float u = k0 * fmaf(0.044715f * x, x * x, x);
    return 0.5f * x * (1.0f + tanh_approx(u));
}

// Eight fp32 accumulator values -> eight bf16 (16 bytes), with the epilogue activation.
__device__ __forceinline__ uint4 pack8_act(const uint32_t* v, int act) {
    float f[8];
#pragma unroll
    for (int j = 0; j < 8; ++j) f[j] = act ? gelu_tanh(__uint_as_float(v[j])) : __uint_as_float(v[j]);
    return make_uint4(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]), pack_bf16x2(f[4], f[5]),
                      pack_bf16x2(f[6], f[7]));
}

template <bool kBf16, int kNT>
struct Cfg {
    static constexpr uint32_t kEBytes = kNT * kKBlock * 2;
    static constexpr uint32_t kLBytes = kTileM * kKBlock * (kBf16 ? 2 : 4);
    static constexpr uint32_t kPBytes = kBf16 ? 0 : kTileM * kKBlock * 2;  // bf16 writes p in place
    static constexpr uint32_t kStageBytes = kEBytes + kLBytes + kPBytes;
    static constexpr int kStagesFit = static_cast<int>((200u * 1024u) / kStageBytes);
    static constexpr int kStages = kStagesFit > 6 ? 6 : kStagesFit;
    static constexpr uint32_t kBarrierBytes = 256;
    static constexpr uint32_t kSmemBytes = kStages * kStageBytes + kBarrierBytes + 1024;
    static_assert(kStages >= 2, "pipeline needs two stages");
    static_assert(kEBytes % 1024 == 0 && kLBytes % 1024 == 0 && kPBytes % 1024 == 0, "1 KB-aligned stage parts");
};

// ------------------------------------------------------------------------------------ PTX wrappers
// Per-CTA wait control in shared memory: the abort flag every wait watches, and the wait limit.
struct WaitCtl {
    int abort;
    int pad;
    long long limit;  // cycles
};
__device__ __forceinline__ bool aborted(const WaitCtl* c) { return *reinterpret_cast<const volatile int*>(&c->abort) != 0; }

// Wait for the phase with the given parity to complete.  Gives up (returning false) when another
// thread of the CTA has aborted or after ctl->limit cycles, recording the expiry.  The first probe
// is inlined at every call site; only a phase not yet complete pays for the out-of-line loop.
__device__ __noinline__ bool mbar_wait_loop(uint64_t* bar, uint32_t parity, WaitCtl* ctl) {
    const long long t0 = clock64();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (aborted(ctl)) return false;
        if (clock64() - t0 > ctl->limit) {
            *reinterpret_cast<volatile int*>(&ctl->abort) = 1;
            atomicMax(&g_device_error, 1);
            return false;
        }
    }
}
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, WaitCtl* ctl) {
    return mbar_try_wait(bar, parity) || mbar_wait_loop(bar, parity, ctl);
}
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* tm, int32_t c0, int32_t c1, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::
            "r"(smem_u32(dst)),
        "l"(tm), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}
// Barrier among the four warps of one softmax group (named barrier 1 + group, 128 threads) that
// also ORs a flag over them, so that every thread of the group takes the same exit decision (a
// partial arrival would hang).
__device__ __forceinline__ bool softmax_group_sync_or(int group, bool flag) {
    uint32_t r;
    asm volatile(
        "{\n\t.reg .pred p, q;\n\t"
        "setp.ne.u32 p, %1, 0;\n\t"
        "bar.red.or.pred q, %2, %3, p;\n\t"
        "selp.u32 %0, 1, 0, q;\n\t}"
        : "=r"(r)
        : "r"(static_cast<uint32_t>(flag)), "r"(1 + group), "n"(kGroupThreads)
        : "memory");
    return r != 0;
}
__device__ __forceinline__ void tcgen05_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tcgen05_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// UMMA shared-memory matrix descriptor: start address, leading / stride byte offsets (16-byte
// units), descriptor version 1 (sm_100), swizzle mode in bits 61..63 (2 = 128 B, 4 = 64 B).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo_bytes, uint32_t sbo_bytes, uint32_t layout) {
    uint64_t d = static_cast<uint64_t>((addr >> 4) & 0x3FFFu);
    d |= static_cast<uint64_t>((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= static_cast<uint64_t>((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= static_cast<uint64_t>(1) << 46;
    d |= static_cast<uint64_t>(layout & 7u) << 61;
    return d;
}
constexpr uint32_t kLayoutSw128 = 2;

// Instruction descriptor for kind::f16: fp32 accumulator, bf16 A and B, A K-major, B MN-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N) {
    return (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) | (static_cast<uint32_t>(N >> 3) << 17) |
           (static_cast<uint32_t>(M >> 4) << 24);
}

__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                          uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&v)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7]),
          "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), "=r"(v[14]), "=r"(v[15]),
          "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]), "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]),
          "=r"(v[24]), "=r"(v[25]), "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// p for 8 consecutive bf16 logits held in one 16-byte chunk, packed back as 8 bf16.
__device__ __forceinline__ uint4 softmax_chunk_bf16(uint4 c, float a, float nb) {
    uint4 o;
    o.x = pack_bf16x2(ex2_approx(fmaf(bf16_lo(c.x), a, nb)), ex2_approx(fmaf(bf16_hi(c.x), a, nb)));
    o.y = pack_bf16x2(ex2_approx(fmaf(bf16_lo(c.y), a, nb)), ex2_approx(fmaf(bf16_hi(c.y), a, nb)));
    o.z = pack_bf16x2(ex2_approx(fmaf(bf16_lo(c.z), a, nb)), ex2_approx(fmaf(bf16_hi(c.z), a, nb)));
    o.w = pack_bf16x2(ex2_approx(fmaf(bf16_lo(c.w), a, nb)), ex2_approx(fmaf(bf16_hi(c.w), a, nb)));
    return o;
}
__device__ __forceinline__ uint32_t softmax_pair_f32(uint32_t x, uint32_t y, float a, float nb) {
    return pack_bf16x2(ex2_approx(fmaf(__uint_as_float(x), a, nb)), ex2_approx(fmaf(__uint_as_float(y), a, nb)));
}

// Turn one logits row of the stage tile into p = exp2(l * a + nb) as the bf16 K-major A operand.
// Rows are 128 bytes with the 128-byte swizzle: 16-byte chunk j of row r sits at j ^ (r & 7).
// bf16 logits are converted in place; fp32 logits arrive as two [128 x 32] sub-tiles and p goes
// to the separate bf16 tile `pt`.
template <bool kBf16>
__device__ __forceinline__ void softmax_row(uint8_t* lt, uint8_t* pt, int row, float a, float nb) {
    const int sw = row & 7;
    if (kBf16) {
        uint8_t* rb = lt + row * 128;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            uint4* q = reinterpret_cast<uint4*>(rb + ((j ^ sw) << 4));
            *q = softmax_chunk_bf16(*q, a, nb);
        }
    } else {
        uint8_t* pb = pt + row * 128;
#pragma unroll
        for (int q = 0; q < 8; ++q) {
            const uint8_t* rb = lt + (q >> 2) * (kTileM * 128) + row * 128;
            const int c = 2 * (q & 3);
            const uint4 c0 = *reinterpret_cast<const uint4*>(rb + ((c ^ sw) << 4));
            const uint4 c1 = *reinterpret_cast<const uint4*>(rb + (((c + 1) ^ sw) << 4));
            uint4 o;
            o.x = softmax_pair_f32(c0.x, c0.y, a, nb);
            o.y = softmax_pair_f32(c0.z, c0.w, a, nb);
            o.z = softmax_pair_f32(c1.x, c1.y, a, nb);
            o.w = softmax_pair_f32(c1.z, c1.w, a, nb);
            *reinterpret_cast<uint4*>(pb + ((q ^ sw) << 4)) = o;
        }
    }
}

// Logits tile copy of one stage: one box of 64 bf16 ids, or two boxes of 32 fp32 ids.
template <bool kBf16>
__device__ __forceinline__ void load_logits_tile(uint8_t* dst, const CUtensorMap* tm, int32_t k0, int32_t row0,
                                                 uint64_t* bar) {
    tma_load_2d(dst, tm, k0, row0, bar);
    if (!kBf16) tma_load_2d(dst + kTileM * 128, tm, k0 + 32, row0, bar);
}

template <bool kBf16, int kNT>
__global__ void __launch_bounds__(kThreads, 1) selfcond_kernel(const __grid_constant__ KernelParams p) {
    using G = Cfg<kBf16, kNT>;
    constexpr int kStages = G::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* efull = reinterpret_cast<uint64_t*>(smem + kStages * G::kStageBytes);
    uint64_t* lfull = efull + kStages;
    uint64_t* pready = lfull + kStages;
    uint64_t* empty = pready + kStages;
    uint64_t* accum = empty + kStages;
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
    WaitCtl* wc = reinterpret_cast<WaitCtl*>(tmem_slot + 2);

    int bid = blockIdx.x;
    const int split = bid % p.splits;
    bid /= p.splits;
    const int nt = bid % p.n_tiles;
    const int mt = bid / p.n_tiles;
    // Split s takes the kKBlock-id blocks s, s + S, s + 2S, ...: at any moment all CTAs read the same
    // few rows of E, so every E row is fetched by all its readers within a short window.
    const int kb0 = split;
    const int kstride = p.splits;
    const int nkb = (p.total_kb - split + p.splits - 1) / p.splits;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&efull[s], 1);
            mbar_init(&lfull[s], 1);
            mbar_init(&pready[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(accum, 1);
        wc->abort = 0;
        wc->limit = p.wait_limit;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(static_cast<uint32_t>(kNT))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
    }
    tcgen05_before_sync();
    __syncthreads();
    tcgen05_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- TMA producer
        if (lane == 0) {
            int issued = 0;
            // a plain operand may be the preceding grid's output (the FFW's hidden layer): wait for it
            // (a no-op unless this is a programmatic dependent launch)
            if (p.plain) grid_dependency_wait();
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                if (!mbar_wait(&empty[s], ph ^ 1, wc)) break;
                uint8_t* st = smem + s * G::kStageBytes;
                const int32_t k0 = (kb0 + i * kstride) * kKBlock;
                mbar_arrive_expect_tx(&lfull[s], G::kLBytes);
                load_logits_tile<kBf16>(st + G::kEBytes, &p.tm_logits, k0, mt * kTileM, &lfull[s]);
                if (kb0 + i * kstride != p.fault_block) {
                    mbar_arrive_expect_tx(&efull[s], G::kEBytes);
#pragma unroll
                    for (int b = 0; b < kNT / 64; ++b)
                        tma_load_2d(st + b * (64 * kKBlock * 2), &p.tm_E, nt * kNT + 64 * b, k0, &efull[s]);
                }
                issued = i + 1;
            }
            if (aborted(wc)) {
                // let the copies already issued land before the CTA's shared memory goes away
                const long long t0 = clock64();  // one deadline for the whole drain
                for (int i = issued - kStages > 0 ? issued - kStages : 0; i < issued; ++i) {
                    const int s = i % kStages;
                    const uint32_t ph = (i / kStages) & 1;
                    const bool e_issued = kb0 + i * kstride != p.fault_block;
                    while (!(mbar_try_wait(&lfull[s], ph) && (!e_issued || mbar_try_wait(&efull[s], ph))) &&
                           clock64() - t0 < wc->limit) {
                    }
                }
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer
        if (lane == 0) {
            constexpr int kMmaN = kNT > 256 ? 256 : kNT;
            constexpr uint32_t idesc = idesc_bf16(kTileM, kMmaN);
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                if (!mbar_wait(&efull[s], ph, wc)) break;
                // plain operands are used as loaded: no softmax hand-off
                if (!mbar_wait(p.plain ? &lfull[s] : &pready[s], ph, wc)) break;
                tcgen05_after_sync();
                uint8_t* st = smem + s * G::kStageBytes;
                const uint32_t a_base = smem_u32(st + G::kEBytes + (kBf16 ? 0 : G::kLBytes));
                const uint32_t b_base = smem_u32(st);
#pragma unroll
                for (int ks = 0; ks < kKBlock / 16; ++ks) {
                    // A: 128 rows x 16 ids, K-major, rows of 128 bytes, 8-row atoms of 1 KB
                    const uint64_t adesc = smem_desc(a_base + ks * 32, 16, 1024, kLayoutSw128);
#pragma unroll
                    for (int nh = 0; nh < kNT / kMmaN; ++nh) {
                        // B: 16 ids x kMmaN columns, MN-major, 64-column boxes 4 KB apart, 8-id atoms of 1 KB
                        const uint64_t bdesc =
                            smem_desc(b_base + nh * (kMmaN / 64) * (64 * kKBlock * 2) + ks * 2048, 64 * kKBlock * 2,
                                      1024, kLayoutSw128);
                        umma_bf16(tmem + nh * kMmaN, adesc, bdesc, idesc, (i > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                umma_commit(&empty[s]);
            }
            umma_commit(accum);
        }
    } else {
        // ---------------------------------------------------------------- softmax + epilogue
        const int quarter = warp & 3;  // TMEM lanes this warp may access: 32 * quarter ..
        const int group = (warp - 2) >> 2;
        const int row = quarter * 32 + lane;
        const int32_t r = mt * kTileM + row;
        const bool valid = r < p.R;
        const float it = valid && !p.plain ? p.inv_tau[r / p.C] : 1.0f;
        const float a = it * kLog2e;
        grid_dependency_wait();  // lse comes from the preceding logits pass (a dependent launch)
        const float nb = valid && !p.plain ? -p.lse[r] * kLog2e : 0.0f;
        for (int i = group; i < (p.plain ? 0 : nkb); i += 2) {  // plain operands need no softmax
            const int s = i % kStages;
            const uint32_t ph = (i / kStages) & 1;
            const bool ok = mbar_wait(&lfull[s], ph, wc);
            uint8_t* lt = smem + s * G::kStageBytes + G::kEBytes;
            if (ok && !p.plain) softmax_row<kBf16>(lt, lt + G::kLBytes, row, a, nb);
            fence_proxy_async_smem();  // each thread's p stores, visible to the tensor core
            if (softmax_group_sync_or(group, !ok)) break;
            if (threadIdx.x == 64 + group * kGroupThreads) mbar_arrive(&pready[s]);
        }
        const bool acc_ok = __all_sync(0xffffffffu, mbar_wait(accum, 0, wc));
        grid_launch_dependents();  // the split sum may launch; it waits for this grid's partials
        if (acc_ok) {
            tcgen05_after_sync();
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            for (int c = group * (kNT / 2); c < (group + 1) * (kNT / 2); c += 32) {
                uint32_t v[32];
                tmem_ld_32x32b_x32(lane_base + c, v);
                if (valid) {
                    const int32_t col = nt * kNT + c;
                    if (p.splits == 1) {
                        uint4* dst = reinterpret_cast<uint4*>(p.z + static_cast<size_t>(r) * p.d + col);
#pragma unroll
                        for (int q = 0; q < 4; ++q) dst[q] = pack8_act(v + 8 * q, p.act);
                    } else {
                        float4* dst = reinterpret_cast<float4*>(
                            p.partial + (static_cast<size_t>(split) * p.R + r) * p.d + col);
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            dst[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]),
                                                 __uint_as_float(v[4 * q + 2]), __uint_as_float(v[4 * q + 3]));
                    }
                }
            }
        }
    }

    tcgen05_before_sync();
    __syncthreads();
    tcgen05_after_sync();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(static_cast<uint32_t>(kNT))
                     : "memory");
}

// ------------------------------------------------------------------------------------ CTA-pair form
// For 129 rows or more, a cluster of two CTAs shares each tile: tcgen05.mma.cta_group::2 with
// M = 256 reads A (p) from both CTAs -- 128 rows each, from their own shared memory -- and B (E)
// split by columns: each CTA stages only the half of every 256-column block that belongs to it,
// so per stage of kKBlock ids a CTA loads half of the tile's E bytes and the rings get deeper.
// The pair's accumulator is 128 TMEM lanes x kNT columns in each CTA (its own rows).
// Signalling: both CTAs' E copies complete on the leader CTA's barrier (cta_group::2 TMA, no
// multicast); the peer's softmax warps arrive remotely on the leader's p-ready barrier; the
// leader's MMA thread commits each stage to its own and to its peer's empty barrier.

template <bool kBf16, int kNT>
struct PairCfg {
    static constexpr int kMmaN = kNT > 256 ? 256 : kNT;
    static constexpr int kBoxesPerHalf = kMmaN / 128;  // 64-column boxes per CTA per MMA block
    static constexpr uint32_t kEBytes = (kNT / 2) * kKBlock * 2;
    static constexpr uint32_t kLBytes = kTileM * kKBlock * (kBf16 ? 2 : 4);
    static constexpr uint32_t kPBytes = kBf16 ? 0 : kTileM * kKBlock * 2;
    static constexpr uint32_t kLStageBytes = kLBytes + kPBytes;
    // A logits stage makes a long round trip (land, softmax, forward to the leader, MMA, release),
    // so the logits ring needs about as much depth as the E ring even though its copies are fast.
    static constexpr uint32_t kBudget = 212u * 1024u;
    static constexpr int kLStagesFit = static_cast<int>((kBudget - 4 * kEBytes) / kLStageBytes);
    static constexpr int kLStages = kLStagesFit > 8 ? 8 : kLStagesFit;
    static constexpr int kEStagesFit = static_cast<int>((kBudget - kLStages * kLStageBytes) / kEBytes);
    static constexpr int kEStages = kEStagesFit > 16 ? 16 : kEStagesFit;
    static constexpr uint32_t kBarrierBytes = 1024;
    static constexpr uint32_t kRingBytes = kEStages * kEBytes + kLStages * kLStageBytes;
    static constexpr uint32_t kSmemBytes = kRingBytes + kBarrierBytes + 1024;
    // epilogue: each of the two epilogue groups stages up to kSlabsPerGroup 16 KB slabs in the
    // drained rings
    static constexpr int kSlabsFit = static_cast<int>(kRingBytes / 2 / 16384u);
    static constexpr int kSlabsPerGroup = kSlabsFit > 8 ? 8 : kSlabsFit;
    static_assert(kSlabsPerGroup >= 1, "the rings must hold one epilogue slab per group");
    static_assert(kNT >= 128 && kNT % 128 == 0, "pair tiles hold whole 64-column boxes per CTA");
    static_assert(kEStages >= 4 && kLStages >= 2, "pipelines need depth");
    static_assert(kEBytes % 1024 == 0 && kLBytes % 1024 == 0 && kPBytes % 1024 == 0, "1 KB-aligned stage parts");
};

constexpr int kPairThreads = 96 + 32 * kNumSoftmaxWarps;  // E producer, MMA/forwarder, logits producer

__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}
// Address of the same shared-memory location in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(uint32_t smem_addr, uint32_t rank) {
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
    return r;
}
__device__ __forceinline__ void cluster_sync() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
// Arrival on a barrier of another CTA of the cluster (default release semantics).
__device__ __forceinline__ void mbar_arrive_remote(uint32_t cluster_addr) {
    asm volatile("mbarrier.arrive.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
// E box copy whose completion is counted on the pair leader's barrier.
__device__ __forceinline__ void tma_load_2d_pair(void* dst, const CUtensorMap* tm, int32_t c0, int32_t c1,
                                                 uint32_t leader_bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, "
        "%3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(tm), "r"(c0), "r"(c1), "r"(leader_bar)
        : "memory");
}
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                               uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}
__device__ __forceinline__ void umma_commit_pair(uint32_t cluster_bar) {
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(cluster_bar)
                 : "memory");
}
// One commit that arrives on the barrier at the same shared-memory offset in both CTAs of the pair
// (own_bar: the executing CTA's shared-memory address of it).
__device__ __forceinline__ void umma_commit_pair_both(uint32_t own_bar) {
    const uint16_t mask = 0x3;
    asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
                 ::"r"(own_bar), "h"(mask)
                 : "memory");
}

// Bulk tensor stores (shared memory -> global; completion tracked by bulk groups).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* tm, int32_t c0, int32_t c1, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(tm), "r"(c0),
                 "r"(c1), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void tma_store_3d(const CUtensorMap* tm, int32_t c0, int32_t c1, int32_t c2, uint32_t src) {
    asm volatile("cp.async.bulk.tensor.3d.global.shared::cta.bulk_group [%0, {%1, %2, %3}], [%4];" ::"l"(tm), "r"(c0),
                 "r"(c1), "r"(c2), "r"(src)
                 : "memory");
}
__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }
// Barrier among the four warps of one epilogue group (named barrier 3 + group, 128 threads).
__device__ __forceinline__ void epilogue_group_bar(int group) {
    asm volatile("bar.sync %0, 128;" ::"r"(3 + group) : "memory");
}
__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint4 v) {
    asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
                 : "memory");
}

// Epilogue of a CTA's 128-row accumulator by one group of four warps (all 128 rows, the group's half
// of the kNT columns): TMEM -> registers -> activation and rounding -> shared memory -> TMA store.
// A slab is 128 rows x 128 bytes (64 bf16 or 32 fp32 columns) in the 128-byte swizzle (16-byte
// chunk c of row r at chunk position c ^ (r & 7)), so each warp's 16-byte stores spread over all
// banks.  The group stages up to kSlabs slabs at a time in its part of the drained stage rings
// (`area`), and its first thread (`issuer`) issues their stores.  Rows past R are clipped by the
// tensor map; a CTA whose rows all lie past R stores nothing.
template <int kNT, int kSlabs>
__device__ void store_tile(const KernelParams& p, uint32_t tmem_lane_base, uint8_t* area, int group, int row,
                           bool issuer, int32_t row0, int32_t col0, int split) {
    constexpr int kHalf = kNT / 2;
    const bool bf16_out = p.splits == 1;
    const int cols_per_slab = bf16_out ? 64 : 32;
    const int n_slabs = kHalf / cols_per_slab;
    const uint32_t area_u32 = smem_u32(area);
    const uint32_t row_base = area_u32 + static_cast<uint32_t>(row) * 128u;
    const uint32_t sw = static_cast<uint32_t>(row & 7);
    for (int b0 = 0; b0 < n_slabs; b0 += kSlabs) {
        const int nb = min(kSlabs, n_slabs - b0);
        if (b0 > 0) {  // the previous batch must have been read out before its slabs are overwritten
            if (issuer) bulk_wait_read_all();
            epilogue_group_bar(group);
        }
        for (int c = b0 * cols_per_slab; c < (b0 + nb) * cols_per_slab; c += 32) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tmem_lane_base + static_cast<uint32_t>(group * kHalf + c), v);
            const uint32_t slab_row = row_base + static_cast<uint32_t>(c / cols_per_slab - b0) * 16384u;
            if (bf16_out) {
                const uint32_t k0 = static_cast<uint32_t>((c % 64) / 8);
#pragma unroll
                for (int k = 0; k < 4; ++k)
                    st_shared_v4(slab_row + (((k0 + static_cast<uint32_t>(k)) ^ sw) << 4), pack8_act(v + 8 * k, p.act));
            } else {
#pragma unroll
                for (int k = 0; k < 8; ++k)
                    st_shared_v4(slab_row + ((static_cast<uint32_t>(k) ^ sw) << 4),
                                 make_uint4(v[4 * k], v[4 * k + 1], v[4 * k + 2], v[4 * k + 3]));
            }
        }
        fence_proxy_async_smem();  // this thread's stores, visible to the bulk copies
        epilogue_group_bar(group);
        if (issuer && row0 < p.R) {
            for (int j = 0; j < nb; ++j) {
                const int32_t col = col0 + group * kHalf + (b0 + j) * cols_per_slab;
                const uint32_t src = area_u32 + static_cast<uint32_t>(j) * 16384u;
                if (!DG_CHECKED(g_device_error, col >= 0 && col + cols_per_slab <= p.d)) continue;
                if (bf16_out)
                    tma_store_2d(&p.tm_out, col, row0, src);
                else
                    tma_store_3d(&p.tm_out, col, row0, split, src);
            }
            bulk_commit();
        }
    }
    if (issuer) bulk_wait_all();  // complete before the CTA may exit
}

template <bool kBf16, int kNT>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kPairThreads, 1)
    selfcond_pair_kernel(const __grid_constant__ KernelParams p) {
    using G = PairCfg<kBf16, kNT>;
    constexpr int kES = G::kEStages, kLS = G::kLStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint8_t* ering = smem;                             // kES x E half-tiles
    uint8_t* lring = smem + kES * G::kEBytes;          // kLS x (logits tile [+ p tile])
    uint64_t* efull = reinterpret_cast<uint64_t*>(lring + kLS * G::kLStageBytes);  // leader's: both halves
    uint64_t* eempty = efull + kES;                    // own E stage free (leader's commit)
    uint64_t* lfull = eempty + kES;                    // own logits landed
    uint64_t* lempty = lfull + kLS;                    // own logits/p stage free (leader's commit)
    uint64_t* pready = lempty + kLS;                   // leader: both CTAs' p; peer: own p (forwarded)
    uint64_t* accum = pready + kLS;                    // own accumulator final
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);
    WaitCtl* wc = reinterpret_cast<WaitCtl*>(tmem_slot + 2);

    const uint32_t rank = cluster_rank();
    int bid = blockIdx.x >> 1;  // pair index
    const int split = bid % p.splits;
    bid /= p.splits;
    const int nt = bid % p.n_tiles;
    const int mp = bid / p.n_tiles;  // rows 256 mp .. 256 mp + 255; this CTA: 128 of them
    // Split s takes the kKBlock-id blocks s, s + S, s + 2S, ...: at any moment all CTAs read the same
    // few rows of E, so every E row is fetched by all its readers within a short window.
    const int kb0 = split;
    const int kstride = p.splits;
    const int nkb = (p.total_kb - split + p.splits - 1) / p.splits;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    constexpr int kFirstSoftmaxWarp = 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kES; ++s) {
            mbar_init(&efull[s], 1);
            mbar_init(&eempty[s], 1);
        }
        for (int s = 0; s < kLS; ++s) {
            mbar_init(&lfull[s], 1);
            mbar_init(&lempty[s], 1);
            mbar_init(&pready[s], rank == 0 ? 2 : 1);
        }
        mbar_init(accum, 1);
        wc->abort = 0;
        wc->limit = p.wait_limit;
        fence_barrier_init();
    }
    if (warp == 1) {
        asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                     "r"(static_cast<uint32_t>(kNT))
                     : "memory");
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
    }
    tcgen05_before_sync();
    cluster_sync();  // barriers of both CTAs initialised before any remote arrival
    tcgen05_after_sync();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ---------------------------------------------------------------- E producer (both CTAs)
        if (lane == 0) {
            const uint32_t leader_efull0 = map_to_rank(smem_u32(&efull[0]), 0);
            int issued = 0;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kES;
                const uint32_t ph = (i / kES) & 1;
                if (!mbar_wait(&eempty[s], ph ^ 1, wc)) break;
                const int32_t k0 = (kb0 + i * kstride) * kKBlock;
                issued = i + 1;
                if (kb0 + i * kstride == p.fault_block) continue;
                if (rank == 0) mbar_arrive_expect_tx(&efull[s], 2 * G::kEBytes);
                uint8_t* dst = ering + s * G::kEBytes;
#pragma unroll
                for (int nh = 0; nh < kNT / G::kMmaN; ++nh)
#pragma unroll
                    for (int j = 0; j < G::kBoxesPerHalf; ++j) {
                        const int col = nt * kNT + nh * G::kMmaN + static_cast<int>(rank) * (G::kMmaN / 2) + 64 * j;
                        DG_CHECK(g_device_error, col + 64 <= p.d && k0 < p.V);
                        tma_load_2d_pair(dst + (nh * G::kBoxesPerHalf + j) * (64 * kKBlock * 2), &p.tm_E, col, k0,
                                         leader_efull0 + s * 8);
                    }
            }
            if (aborted(wc) && rank == 0) {
                // both halves of the last stages land on the leader's barriers: wait for them (bounded)
                const long long t0 = clock64();  // one deadline for the whole drain
                for (int i = issued - kES > 0 ? issued - kES : 0; i < issued; ++i) {
                    if (kb0 + i * kstride == p.fault_block) continue;
                    while (!mbar_try_wait(&efull[i % kES], (i / kES) & 1) && clock64() - t0 < wc->limit) {
                    }
                }
            }
        }
    } else if (warp == 2) {
        // ---------------------------------------------------------------- logits producer (both CTAs)
        if (lane == 0) {
            int issued = 0;
            // Plain operands (bf16, used as loaded): both CTAs' tiles complete on the leader's barrier,
            // which the MMA thread waits on directly.
            const uint32_t leader_lfull0 = map_to_rank(smem_u32(&lfull[0]), 0);
            // a plain operand may be the preceding grid's output (the FFW's hidden layer): wait for it
            // (a no-op unless this is a programmatic dependent launch); the E copies need no wait
            if (p.plain) grid_dependency_wait();
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kLS;
                const uint32_t ph = (i / kLS) & 1;
                if (!mbar_wait(&lempty[s], ph ^ 1, wc)) break;
                const int32_t k0 = (kb0 + i * kstride) * kKBlock;
                const int32_t row0 = mp * 2 * kTileM + static_cast<int>(rank) * kTileM;
                if (kBf16 && p.plain) {
                    if (rank == 0) mbar_arrive_expect_tx(&lfull[s], 2 * G::kLBytes);
                    tma_load_2d_pair(lring + s * G::kLStageBytes, &p.tm_logits, k0, row0, leader_lfull0 + s * 8);
                } else {
                    mbar_arrive_expect_tx(&lfull[s], G::kLBytes);
                    load_logits_tile<kBf16>(lring + s * G::kLStageBytes, &p.tm_logits, k0, row0, &lfull[s]);
                }
                issued = i + 1;
            }
            if (aborted(wc) && (!p.plain || rank == 0)) {
                const long long t0 = clock64();  // one deadline for the whole drain
                for (int i = issued - kLS > 0 ? issued - kLS : 0; i < issued; ++i) {
                    while (!mbar_try_wait(&lfull[i % kLS], (i / kLS) & 1) && clock64() - t0 < wc->limit) {
                    }
                }
            }
        }
    } else if (warp == 1 && rank == 1) {
        // ---------------------------------------------------------------- p-ready forwarder (peer)
        // Passes "p of stage s is written" on to the leader, off the softmax warps' critical path.
        if (lane == 0) {
            const uint32_t leader_pready0 = map_to_rank(smem_u32(&pready[0]), 0);
            for (int i = 0; i < (p.plain ? 0 : nkb); ++i) {
                const int s = i % kLS;
                if (!mbar_wait(&pready[s], (i / kLS) & 1, wc)) break;
                mbar_arrive_remote(leader_pready0 + s * 8);
            }
        }
    } else if (warp == 1) {
        // ---------------------------------------------------------------- MMA issuer (leader)
        if (lane == 0) {
            constexpr uint32_t idesc = idesc_bf16(2 * kTileM, G::kMmaN);
            for (int i = 0; i < nkb; ++i) {
                const int es = i % kES, ls = i % kLS;
                if (!mbar_wait(&efull[es], (i / kES) & 1, wc)) break;
                if (!mbar_wait(p.plain ? &lfull[ls] : &pready[ls], (i / kLS) & 1, wc)) break;
                tcgen05_after_sync();
                const uint32_t a_base = smem_u32(lring + ls * G::kLStageBytes + (kBf16 ? 0 : G::kLBytes));
                const uint32_t b_base = smem_u32(ering + es * G::kEBytes);
#pragma unroll
                for (int ks = 0; ks < kKBlock / 16; ++ks) {
                    const uint64_t adesc = smem_desc(a_base + ks * 32, 16, 1024, kLayoutSw128);
#pragma unroll
                    for (int nh = 0; nh < kNT / G::kMmaN; ++nh) {
                        const uint64_t bdesc = smem_desc(
                            b_base + nh * G::kBoxesPerHalf * (64 * kKBlock * 2) + ks * 2048, 64 * kKBlock * 2, 1024,
                            kLayoutSw128);
                        umma_bf16_pair(tmem + nh * G::kMmaN, adesc, bdesc, idesc, (i > 0 || ks > 0) ? 1u : 0u);
                    }
                }
                umma_commit_pair_both(smem_u32(&eempty[es]));
                umma_commit_pair_both(smem_u32(&lempty[ls]));
            }
            umma_commit_pair(map_to_rank(smem_u32(accum), 0));
            umma_commit_pair(map_to_rank(smem_u32(accum), 1));
        }
    } else {
        // ---------------------------------------------------------------- softmax + epilogue (both CTAs)
        const int quarter = warp & 3;  // TMEM lanes this warp may access
        const int group = (warp - kFirstSoftmaxWarp) >> 2;
        const int row = quarter * 32 + lane;
        const int32_t r = mp * 2 * kTileM + static_cast<int>(rank) * kTileM + row;
        const bool valid = r < p.R;
        const float it = valid && !p.plain ? p.inv_tau[r / p.C] : 1.0f;
        const float a = it * kLog2e;
        grid_dependency_wait();  // lse comes from the preceding logits pass (a dependent launch)
        const float nb = valid && !p.plain ? -p.lse[r] * kLog2e : 0.0f;
        const int leader_thread = (kFirstSoftmaxWarp + 4 * group) * 32;
        for (int i = group; i < (p.plain ? 0 : nkb); i += 2) {  // plain operands need no softmax
            const int s = i % kLS;
            const bool ok = mbar_wait(&lfull[s], (i / kLS) & 1, wc);
            uint8_t* lt = lring + s * G::kLStageBytes;
            if (ok && !p.plain) softmax_row<kBf16>(lt, lt + G::kLBytes, row, a, nb);
            fence_proxy_async_smem();  // each thread's p stores, visible to the tensor core
            if (softmax_group_sync_or(group, !ok)) break;
            if (static_cast<int>(threadIdx.x) == leader_thread) mbar_arrive(&pready[s]);
        }
        // one exit decision per group: its warps meet at named barriers in the epilogue
        const bool acc_fail = softmax_group_sync_or(group, !mbar_wait(accum, 0, wc));
        grid_launch_dependents();  // the split sum may launch; it waits for this grid's partials
        if (!acc_fail) {
            tcgen05_after_sync();
            const uint32_t lane_base = tmem + (static_cast<uint32_t>(quarter * 32) << 16);
            const int32_t row0 = mp * 2 * kTileM + static_cast<int>(rank) * kTileM;
            store_tile<kNT, G::kSlabsPerGroup>(p, lane_base, smem + group * G::kSlabsPerGroup * 16384, group, row,
                                               static_cast<int>(threadIdx.x) == leader_thread, row0, nt * kNT, split);
        }
    }

    // Neither CTA leaves (or frees TMEM) while its peer may still touch its shared memory or the
    // pair's accumulator.
    tcgen05_before_sync();
    __syncthreads();
    cluster_sync();
    tcgen05_after_sync();
    if (warp == 1)
        asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(static_cast<uint32_t>(kNT))
                     : "memory");
}

// Test of the bounded wait itself: one thread waits on a barrier that nothing will ever arrive on.
// The wait gives up after `limit` cycles, records device error 1 and the kernel returns normally.
__global__ void bounded_wait_test_kernel(long long limit) {
    __shared__ __align__(8) uint64_t bar;
    __shared__ WaitCtl wc;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        wc.abort = 0;
        wc.limit = limit;
        fence_barrier_init();
    }
    __syncthreads();
    if (threadIdx.x == 0) mbar_wait(&bar, 0, &wc);
    __syncthreads();
}

// z[i] = bf16(sum_s partial[s][i]) in a fixed order (deterministic).
// Few splits (the FFW's first layer has two): each thread takes kPos positions a stride apart and
// issues all their loads before the first add, so a thread's positions cost one memory round trip.
template <int kPos, int kMaxS>
__global__ void __launch_bounds__(256) splitk_reduce_few_kernel(const float4* __restrict__ partial,
                                                                uint2* __restrict__ z, int64_t n4, int splits,
                                                                int act) {
    grid_dependency_wait();  // launched dependent on the contraction: its partials must be complete
    grid_launch_dependents();  // a dependent (the FFW's second layer) may be placed; it waits for this grid
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    for (int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i0 < n4; i0 += kPos * stride) {
        float4 v[kPos][kMaxS];
#pragma unroll
        for (int q = 0; q < kPos; ++q)
#pragma unroll
            for (int s = 0; s < kMaxS; ++s)
                if (s < splits && i0 + q * stride < n4)
                    v[q][s] = __ldcs(partial + static_cast<int64_t>(s) * n4 + i0 + q * stride);
#pragma unroll
        for (int q = 0; q < kPos; ++q) {
            const int64_t i = i0 + q * stride;
            if (i >= n4) continue;
            float4 acc = v[q][0];  // splits summed in order 0, 1, ... (deterministic)
#pragma unroll
            for (int s = 1; s < kMaxS; ++s)
                if (s < splits) {
                    acc.x += v[q][s].x;
                    acc.y += v[q][s].y;
                    acc.z += v[q][s].z;
                    acc.w += v[q][s].w;
                }
            if (act) {
                acc.x = gelu_tanh(acc.x);
                acc.y = gelu_tanh(acc.y);
                acc.z = gelu_tanh(acc.z);
                acc.w = gelu_tanh(acc.w);
            }
            z[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
        }
    }
}

__global__ void __launch_bounds__(256) splitk_reduce_kernel(const float4* __restrict__ partial, uint2* __restrict__ z,
                                                            int64_t n4, int splits, int act) {
    grid_dependency_wait();  // launched dependent on the contraction: its partials must be complete
    grid_launch_dependents();  // a dependent (the FFW's second layer) may be placed; it waits for this grid
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        // splits summed in order 0, 1, 2, ... (deterministic); loads issued eight at a time
        float4 acc = __ldcs(partial + i);
        int s = 1;
        for (; s + 8 <= splits; s += 8) {
            float4 v[8];
#pragma unroll
            for (int u = 0; u < 8; ++u) v[u] = __ldcs(partial + static_cast<int64_t>(s + u) * n4 + i);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                acc.x += v[u].x;
                acc.y += v[u].y;
                acc.z += v[u].z;
                acc.w += v[u].w;
            }
        }
        for (; s < splits; ++s) {
            const float4 v = __ldcs(partial + static_cast<int64_t>(s) * n4 + i);
            acc.x += v.x;
            acc.y += v.y;
            acc.z += v.z;
            acc.w += v.w;
        }
        if (act) {
            acc.x = gelu_tanh(acc.x);
            acc.y = gelu_tanh(acc.y);
            acc.z = gelu_tanh(acc.z);
            acc.w = gelu_tanh(acc.w);
        }
        z[i] = make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
    }
}

__global__ void convert_f32_bf16_kernel(const float* __restrict__ in, uint16_t* __restrict__ out, int64_t n) {
    for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
         i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
        const __nv_bfloat16 h = __float2bfloat16_rn(in[i]);
        out[i] = *reinterpret_cast<const uint16_t*>(&h);
    }
}

// ------------------------------------------------------------------------------------ host side
using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encoder() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    });
    return fn;
}

cudaError_t encode_2d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, uint64_t inner, uint64_t outer,
                      uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer, CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t dims[2] = {inner, outer};
    const cuuint64_t strides[1] = {row_bytes};
    const cuuint32_t box[2] = {box_inner, box_outer};
    const cuuint32_t estr[2] = {1, 1};
    const CUresult r = fn(tm, dt, 2, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                          sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

cudaError_t encode_3d(CUtensorMap* tm, CUtensorMapDataType dt, const void* base, const uint64_t (&dims)[3],
                      const uint64_t (&strides_bytes)[2], const uint32_t (&box)[3], CUtensorMapSwizzle sw) {
    EncodeTiledFn fn = encoder();
    if (!fn) return cudaErrorNotSupported;
    const cuuint64_t d[3] = {dims[0], dims[1], dims[2]};
    const cuuint64_t st[2] = {strides_bytes[0], strides_bytes[1]};
    const cuuint32_t b[3] = {box[0], box[1], box[2]};
    const cuuint32_t estr[3] = {1, 1, 1};
    const CUresult r = fn(tm, dt, 3, const_cast<void*>(base), d, st, b, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, sw,
                          CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// Column tile: 512 when d allows; fp32 logits (small test workloads) stage twice the bytes per
// tile and use at most 256 columns so that the pipeline keeps its depth.
int pick_ntile(int d, bool logits_bf16) {
    const int nt = d % 512 == 0 ? 512 : d % 256 == 0 ? 256 : d % 128 == 0 ? 128 : 64;
    return logits_bf16 ? nt : (nt > 256 ? 256 : nt);
}


// Work plan: CTA pairs (M = 256 per pair) when there are more than 128 rows and the column tile
// is at least 128 wide, single CTAs otherwise; the vocabulary is split so that the grid is about
// one wave (one CTA per SM).
struct Plan {
    bool pair;
    int m_tiles;   // 128-row tiles (single) or 256-row pair tiles
    int n_tiles;
    int splits;
    int total_kb;
    int ctas;
};

// Plain-operand GEMMs (the feed-forward block) are short in K: 256-column tiles (half the A-operand
// re-reads of 128-column tiles) with a split of K that fills the GPU.
int pick_ntile_plain(int d) { return d % 256 == 0 ? 256 : d % 128 == 0 ? 128 : 64; }

Plan plan(int R, int V, int d, bool logits_bf16, bool plain) {
    Plan pl;
    const int nt = plain ? pick_ntile_plain(d) : pick_ntile(d, logits_bf16);
    pl.pair = R > kTileM && nt >= 128;
    pl.m_tiles = pl.pair ? (R + 2 * kTileM - 1) / (2 * kTileM) : (R + kTileM - 1) / kTileM;
    pl.n_tiles = d / nt;
    pl.total_kb = (V + kKBlock - 1) / kKBlock;
    const int units = pl.m_tiles * pl.n_tiles;
    const int per_unit = pl.pair ? 2 : 1;
    int s = num_sms() / (per_unit * units);
    if (s < 1) s = 1;
    if (s > pl.total_kb) s = pl.total_kb;
    pl.splits = s;
    pl.ctas = per_unit * units * s;
    return pl;
}

// Launch on `st`; with `dependent`, as a programmatic dependent launch of the preceding kernel
// (it may start early; the kernel waits before reading that kernel's outputs).
template <typename Kernel, typename Param>
cudaError_t launch_maybe_dependent(Kernel kernel, int grid, int threads, size_t smem, cudaStream_t st,
                                   const Param& param, bool dependent) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(grid));
    cfg.blockDim = dim3(static_cast<unsigned>(threads));
    cfg.dynamicSmemBytes = smem;
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = dependent ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, param);
}

template <bool kBf16, int kNT>
cudaError_t launch_kernel(const KernelParams& kp, int grid, cudaStream_t st, bool dependent) {
    using G = Cfg<kBf16, kNT>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(selfcond_kernel<kBf16, kNT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                        static_cast<int>(G::kSmemBytes));
    });
    if (attr_err != cudaSuccess) return attr_err;
    return launch_maybe_dependent(selfcond_kernel<kBf16, kNT>, grid, kThreads, G::kSmemBytes, st, kp, dependent);
}

template <bool kBf16, int kNT>
cudaError_t launch_pair_kernel(const KernelParams& kp, int grid, cudaStream_t st, bool dependent) {
    using G = PairCfg<kBf16, kNT>;
    static std::once_flag once;
    static cudaError_t attr_err = cudaSuccess;
    std::call_once(once, [] {
        attr_err = cudaFuncSetAttribute(selfcond_pair_kernel<kBf16, kNT>,
                                        cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(G::kSmemBytes));
    });
    if (attr_err != cudaSuccess) return attr_err;
    return launch_maybe_dependent(selfcond_pair_kernel<kBf16, kNT>, grid, kPairThreads, G::kSmemBytes, st, kp,
                                  dependent);
}

}  // namespace

int num_sms() {
    static std::atomic<int> cached{0};
    int v = cached.load();
    if (v == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0) v = 148;
        cached.store(v);
    }
    return v;
}

size_t selfcond_partial_bytes(int32_t R, int32_t V, int32_t d, bool logits_bf16, bool plain) {
    if (R < 1 || V < 1 || d < 64) return 0;
    const Plan pl = plan(R, V, d, logits_bf16, plain);
    return pl.splits > 1 ? static_cast<size_t>(pl.splits) * R * d * sizeof(float) : 0;
}

cudaError_t launch_selfcond(const SelfcondParams& sp, cudaStream_t st) {
    static thread_local KernelParams kp;
    std::memset(&kp, 0, sizeof(kp));
    const Plan pl = plan(sp.R, sp.V, sp.d, sp.logits_bf16 != 0, sp.plain_a != 0);
    const int splits = pl.splits;
    const int nt = sp.plain_a ? pick_ntile_plain(sp.d) : pick_ntile(sp.d, sp.logits_bf16 != 0);
    cudaError_t e;
    if (sp.logits_bf16)
        e = encode_2d(&kp.tm_logits, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sp.logits, sp.V, sp.R,
                      static_cast<uint64_t>(sp.ld) * 2, kKBlock, kTileM, CU_TENSOR_MAP_SWIZZLE_128B);
    else
        e = encode_2d(&kp.tm_logits, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sp.logits, sp.V, sp.R,
                      static_cast<uint64_t>(sp.ld) * 4, 32, kTileM, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    e = encode_2d(&kp.tm_E, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sp.E, sp.d, sp.V, static_cast<uint64_t>(sp.d) * 2, 64,
                  kKBlock, CU_TENSOR_MAP_SWIZZLE_128B);
    if (e != cudaSuccess) return e;
    if (pl.pair) {  // the pair kernel stores its tiles with TMA: z, or the split's partial sums
        if (splits == 1)
            e = encode_2d(&kp.tm_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, sp.z, sp.d, sp.R, static_cast<uint64_t>(sp.d) * 2,
                          64, kTileM, CU_TENSOR_MAP_SWIZZLE_128B);
        else
            e = encode_3d(&kp.tm_out, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, sp.partial,
                          {static_cast<uint64_t>(sp.d), static_cast<uint64_t>(sp.R), static_cast<uint64_t>(splits)},
                          {static_cast<uint64_t>(sp.d) * 4, static_cast<uint64_t>(sp.R) * sp.d * 4},
                          {32u, static_cast<uint32_t>(kTileM), 1u}, CU_TENSOR_MAP_SWIZZLE_128B);
        if (e != cudaSuccess) return e;
    }
    kp.lse = sp.lse;
    kp.z = sp.z;
    kp.partial = sp.partial;
    kp.R = sp.R;
    kp.C = sp.C;
    kp.V = sp.V;
    kp.d = sp.d;
    kp.n_tiles = pl.n_tiles;
    kp.splits = splits;
    kp.total_kb = pl.total_kb;
    kp.wait_limit = sp.wait_limit > 0 ? sp.wait_limit : kWaitLimitCycles;
    kp.fault_block = sp.fault_block;
    kp.plain = sp.plain_a;
    kp.act = sp.act;
    std::memcpy(kp.inv_tau, sp.inv_tau, sizeof(kp.inv_tau));
    const int grid = pl.ctas;
#define DG_SC(BF, NT) e = launch_kernel<BF, NT>(kp, grid, st, sp.dependent != 0)
#define DG_PC(BF, NT) e = launch_pair_kernel<BF, NT>(kp, grid, st, sp.dependent != 0)
    if (pl.pair) {
        if (sp.logits_bf16) {
            if (nt == 512) DG_PC(true, 512);
            else if (nt == 256) DG_PC(true, 256);
            else DG_PC(true, 128);
        } else {
            if (nt == 256) DG_PC(false, 256);
            else DG_PC(false, 128);
        }
    } else if (sp.logits_bf16) {
        if (nt == 512) DG_SC(true, 512);
        else if (nt == 256) DG_SC(true, 256);
        else if (nt == 128) DG_SC(true, 128);
        else DG_SC(true, 64);
    } else {
        if (nt == 256) DG_SC(false, 256);
        else if (nt == 128) DG_SC(false, 128);
        else DG_SC(false, 64);
    }
#undef DG_SC
#undef DG_PC
    note_launches(1);
    if (e != cudaSuccess || splits == 1) return e;
    const int64_t n4 = static_cast<int64_t>(sp.R) * sp.d / 4;
    const int blocks = static_cast<int>(std::min<int64_t>((n4 + 255) / 256, 4LL * num_sms()));
    // a dependent launch of the contraction: it may start early and waits for the partials
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(blocks));
    cfg.blockDim = dim3(256);
    cfg.stream = st;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (splits == 2)
        e = cudaLaunchKernelEx(&cfg, splitk_reduce_few_kernel<4, 2>, reinterpret_cast<const float4*>(sp.partial),
                               reinterpret_cast<uint2*>(sp.z), n4, splits, static_cast<int>(sp.act));
    else if (splits <= 4)
        e = cudaLaunchKernelEx(&cfg, splitk_reduce_few_kernel<2, 4>, reinterpret_cast<const float4*>(sp.partial),
                               reinterpret_cast<uint2*>(sp.z), n4, splits, static_cast<int>(sp.act));
    else
        e = cudaLaunchKernelEx(&cfg, splitk_reduce_kernel, reinterpret_cast<const float4*>(sp.partial),
                               reinterpret_cast<uint2*>(sp.z), n4, splits, static_cast<int>(sp.act));
    if (e != cudaSuccess) return e;
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_convert_f32_bf16(const float* in, uint16_t* out, int64_t n, cudaStream_t s) {
    const int blocks = static_cast<int>(std::min<int64_t>((n + 255) / 256, 8LL * num_sms()));
    convert_f32_bf16_kernel<<<blocks, 256, 0, s>>>(in, out, n);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t launch_bounded_wait_test(long long limit_cycles, cudaStream_t st) {
    bounded_wait_test_kernel<<<1, 32, 0, st>>>(limit_cycles);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t read_and_clear_device_error(int* out) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int));
    }
    *out = v;
    return e;
}

}  // namespace dg
