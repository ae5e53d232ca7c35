// Logits pass: one streaming read of each logits row, then a per-row merge.
//
// DiffusionGemma Technical Report (hyper.ai summary), section "Method":
//   p0 = Softmax(L_t / tau_t)  and  x_{t-dt} ~ Step(x_t, p0),
// with the forward path kappa_t delta(x_t, x_0) + (1 - kappa_t)/V.  The same pass, with a different
// epilogue, gives the log-sum-exp for the self-conditioning contraction and the canvas
// cross-entropy L = -sum_i log p(x_0^i | ...).
//
// Phase 1 (all CTAs): each warp streams one group of 4 chunks (4 x kChunk = 2048 consecutive ids)
//   of one row with 16-byte non-allocating loads (bf16: 8 loads of 16 B per lane, 512 B per
//   warp-load); each 8-lane subgroup computes its chunk's raw maximum, S = sum exp(l' - m') and
//   T = sum exp(l' - m')(l' - m') with l' = l * inv_tau and m' = max l', and writes one 16-byte
//   record per chunk.
// Phase 2 (merge_kernel, one CTA per row, launched as a programmatic dependent of phase 1 once every
//   phase-1 CTA has started; each merge waits only for its own row, whose streaming CTAs count
//   their records with a release increment and do not wait themselves): merges the row's chunk
//   records into lse, max-prob and entropy, finds the argmax, draws x0_hat by two-level
//   Gumbel-max (level 1 over chunk records, level 2 by re-reading the winning chunk from L2), and
//   samples the Step posterior with one Philox draw.  Rows finish streaming in order, so most
//   merges run while later rows still stream.
#include "common.cuh"
#include "kernels.cuh"

namespace dg {

namespace {

// Device error word of the logits pass: set when a merge's bounded wait expires.
__device__ int g_pass_error = 0;
constexpr long long kMergeWaitLimit = 4000000000LL;  // SM cycles, about 2 s


__device__ __forceinline__ unsigned ld_relaxed_u32(const unsigned* addr) {
    unsigned v;
    asm volatile("ld.relaxed.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(addr) : "memory");
    return v;
}
__device__ __forceinline__ unsigned long long ld_relaxed_u64(const unsigned long long* addr) {
    unsigned long long v;
    asm volatile("ld.relaxed.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(addr) : "memory");
    return v;
}
__device__ __forceinline__ void st_relaxed_u64(unsigned long long* addr, unsigned long long v) {
    asm volatile("st.relaxed.gpu.global.u64 [%0], %1;" ::"l"(addr), "l"(v) : "memory");
}

// Tag of the current call's records, in [1, 65535] (a zeroed workspace holds tag 0).
__device__ __forceinline__ unsigned call_tag(const PassParams& p) { return ld_relaxed_u32(p.epoch) % 65535u + 1u; }

// Chunk records are published without a fence: every 64-bit word carries the call's tag beside its
// value, and an aligned 64-bit store is single-copy atomic, so a reader sees either the previous
// call's word or this call's.  A release per streaming CTA would keep the CTA's slot for a store
// round trip and cost about 2 us over the pass.  Layout, kRecWords words per chunk:
//   bf16 logits: w0 = S << 32 | bf16(m_raw) << 16 | tag,  w1 = tag << 32 | T
//   fp32 logits: w0 = tag << 32 | m_raw,  w1 = tag << 32 | S,  w2 = tag << 32 | T
template <bool kBf16>
__device__ __forceinline__ void put_record(unsigned long long* w, float m_raw, float S, float T, unsigned tag) {
    if (kBf16) {
        st_relaxed_u64(w, static_cast<unsigned long long>(__float_as_uint(S)) << 32 |
                              (__float_as_uint(m_raw) & 0xFFFF0000u) | tag);
        st_relaxed_u64(w + 1, static_cast<unsigned long long>(tag) << 32 | __float_as_uint(T));
    } else {
        const unsigned long long t = static_cast<unsigned long long>(tag) << 32;
        st_relaxed_u64(w, t | __float_as_uint(m_raw));
        st_relaxed_u64(w + 1, t | __float_as_uint(S));
        st_relaxed_u64(w + 2, t | __float_as_uint(T));
    }
}
// Chunk j's record as (m_raw, S, T, -); `ok` is cleared unless every word carries `tag`.
template <bool kBf16>
__device__ __forceinline__ float4 get_record(const unsigned long long* rec, int32_t j, unsigned tag, bool& ok) {
    const unsigned long long* w = rec + static_cast<size_t>(j) * kRecWords;
    if (kBf16) {
        const unsigned long long a = ld_relaxed_u64(w), b = ld_relaxed_u64(w + 1);
        ok &= (static_cast<uint32_t>(a) & 0xFFFFu) == tag && static_cast<uint32_t>(b >> 32) == tag;
        return make_float4(__uint_as_float(static_cast<uint32_t>(a) & 0xFFFF0000u),
                           __uint_as_float(static_cast<uint32_t>(a >> 32)), __uint_as_float(static_cast<uint32_t>(b)),
                           0.f);
    }
    const unsigned long long a = ld_relaxed_u64(w), b = ld_relaxed_u64(w + 1), c = ld_relaxed_u64(w + 2);
    ok &= static_cast<uint32_t>(a >> 32) == tag && static_cast<uint32_t>(b >> 32) == tag &&
          static_cast<uint32_t>(c >> 32) == tag;
    return make_float4(__uint_as_float(static_cast<uint32_t>(a)), __uint_as_float(static_cast<uint32_t>(b)),
                       __uint_as_float(static_cast<uint32_t>(c)), 0.f);
}

// bf16 -1.0e30 (0xF14A), used twice in a 32-bit word: -inf logits are clamped to it so that the
// entropy sum never forms 0 * -inf.
constexpr uint32_t kNegBigBf16x2 = 0xF14AF14Au;
__device__ __forceinline__ float neg_big(bool bf16) {
    return bf16 ? __uint_as_float(0xF14A0000u) : kNegBig;
}

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b) {
    __nv_bfloat162 x = *reinterpret_cast<__nv_bfloat162*>(&a);
    __nv_bfloat162 y = *reinterpret_cast<__nv_bfloat162*>(&b);
    __nv_bfloat162 r = __hmax2(x, y);
    return *reinterpret_cast<uint32_t*>(&r);
}

struct ChunkStats {
    float m_raw;  // max of the (clamped) raw logits in the chunk
    float S;      // sum exp(l' - m'),            m' = m_raw * inv_tau (fp32)
    float T;      // sum exp(l' - m') (l' - m')   (natural-log units)
};

// Reductions over the 8 lanes that share one chunk (lanes 8k .. 8k+7).
__device__ __forceinline__ float max8(float v) {
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
    return v;
}
__device__ __forceinline__ float sum8(float v) {
#pragma unroll
    for (int o = 4; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
    return v;
}

// A chunk whose maximum is the clamp value holds only masked (-inf) logits: its mass is zero.
// The shuffles run on every lane (the mask names the whole warp); only the result is selected.
__device__ __forceinline__ ChunkStats finish(float m_raw, float s, float t, float nbig) {
    ChunkStats cs;
    cs.m_raw = m_raw;
    const float S = sum8(s);
    const float T = sum8(t) * kLn2;
    const bool masked = !(m_raw > nbig);
    cs.S = masked ? 0.f : S;
    cs.T = masked ? 0.f : T;
    return cs;
}

// One full group of 4 chunks (2048 ids) by one warp, bf16.  Lane l owns chunk l / 8 of the group;
// its 8 lanes read the chunk's 1 KB as 8 loads of 16 B, each load instruction covering four
// contiguous 128-byte segments across the warp.
__device__ __forceinline__ ChunkStats group_full_bf16(const char* group, int lane, float inv_tau) {
    const char* chunk = group + (lane >> 3) * (kChunk * 2) + (lane & 7) * 16;
    uint32_t w[32];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
        const uint4 v = ld_stream_v4(chunk + i * 128);
        w[4 * i + 0] = v.x;
        w[4 * i + 1] = v.y;
        w[4 * i + 2] = v.z;
        w[4 * i + 3] = v.w;
    }
    uint32_t mx = kNegBigBf16x2;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        w[i] = bmax2(w[i], kNegBigBf16x2);
        mx = bmax2(mx, w[i]);
    }
    const float m_raw = max8(fmaxf(bf16_lo(mx), bf16_hi(mx)));
    const float a = inv_tau * kLog2e;
    const float nb = -(m_raw * inv_tau) * kLog2e;
    float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) {
        const float x0 = fmaf(bf16_lo(w[i]), a, nb);
        const float x1 = fmaf(bf16_hi(w[i]), a, nb);
        const float e0 = ex2_approx(x0);
        const float e1 = ex2_approx(x1);
        s0 += e0;
        s1 += e1;
        t0 = fmaf(e0, x0, t0);
        t1 = fmaf(e1, x1, t1);
    }
    return finish(m_raw, s0 + s1, t0 + t1, neg_big(true));
}

// Same for fp32: a chunk is 2 KB, 16 loads of 16 B per lane.
__device__ __forceinline__ ChunkStats group_full_f32(const char* group, int lane, float inv_tau) {
    const char* chunk = group + (lane >> 3) * (kChunk * 4) + (lane & 7) * 16;
    float f[64];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const uint4 v = ld_stream_v4(chunk + i * 128);
        f[4 * i + 0] = __uint_as_float(v.x);
        f[4 * i + 1] = __uint_as_float(v.y);
        f[4 * i + 2] = __uint_as_float(v.z);
        f[4 * i + 3] = __uint_as_float(v.w);
    }
    float m = kNegBig;
#pragma unroll
    for (int i = 0; i < 64; ++i) {
        f[i] = fmaxf(f[i], kNegBig);
        m = fmaxf(m, f[i]);
    }
    const float m_raw = max8(m);
    const float a = inv_tau * kLog2e;
    const float nb = -(m_raw * inv_tau) * kLog2e;
    float s0 = 0.f, s1 = 0.f, t0 = 0.f, t1 = 0.f;
#pragma unroll
    for (int i = 0; i < 64; i += 2) {
        const float x0 = fmaf(f[i], a, nb);
        const float x1 = fmaf(f[i + 1], a, nb);
        const float e0 = ex2_approx(x0);
        const float e1 = ex2_approx(x1);
        s0 += e0;
        s1 += e1;
        t0 = fmaf(e0, x0, t0);
        t1 = fmaf(e1, x1, t1);
    }
    return finish(m_raw, s0 + s1, t0 + t1, kNegBig);
}

// A group that runs past V (the ragged tail, or V < 2048): element-wise and bounds-checked; lanes
// whose chunk starts at or past V compute an empty chunk.
__device__ __noinline__ ChunkStats group_ragged(const void* row, bool bf16, int32_t chunk_lo, int32_t V, int lane,
                                               float inv_tau) {
    const float nbig = neg_big(bf16);
    const int32_t lo = chunk_lo + (lane >> 3) * kChunk;
    const int32_t hi = min(lo + kChunk, V);
    float m = nbig;
    for (int32_t v = lo + (lane & 7); v < hi; v += 8) m = fmaxf(m, fmaxf(load_logit(row, v, bf16), nbig));
    const float m_raw = max8(m);
    const float a = inv_tau * kLog2e;
    const float nb = -(m_raw * inv_tau) * kLog2e;
    float s = 0.f, t = 0.f;
    for (int32_t v = lo + (lane & 7); v < hi; v += 8) {
        const float x = fmaf(fmaxf(load_logit(row, v, bf16), nbig), a, nb);
        const float e = ex2_approx(x);
        s += e;
        t = fmaf(e, x, t);
    }
    return finish(m_raw, s, t, nbig);
}

// Four consecutive logits [v, v + 4) of a row as raw words (bf16: 8 bytes, fp32: 16 bytes); one
// vector load when the quad lies inside [.., hi), element loads at the ragged end.
struct RawQuad {
    uint32_t w[4];
};
template <bool kBf16>
__device__ __forceinline__ RawQuad load_quad(const void* row, int32_t v, int32_t hi) {
    RawQuad q;
    if (v + 4 <= hi) {
        if (kBf16) {
            const uint2 x = *reinterpret_cast<const uint2*>(reinterpret_cast<const uint16_t*>(row) + v);
            q.w[0] = x.x;
            q.w[1] = x.y;
            q.w[2] = q.w[3] = 0u;
        } else {
            const uint4 x = *reinterpret_cast<const uint4*>(reinterpret_cast<const float*>(row) + v);
            q.w[0] = x.x;
            q.w[1] = x.y;
            q.w[2] = x.z;
            q.w[3] = x.w;
        }
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) q.w[k] = v + k < hi ? __float_as_uint(load_logit(row, v + k, kBf16)) : 0u;
    }
    return q;
}
// The quad as clamped floats; ids at or past hi are -inf.
template <bool kBf16>
__device__ __forceinline__ void unpack_quad(const RawQuad& q, int32_t v, int32_t hi, float nbig, float (&out)[4]) {
    if (v + 4 <= hi && kBf16) {
        out[0] = bf16_lo(q.w[0]);
        out[1] = bf16_hi(q.w[0]);
        out[2] = bf16_lo(q.w[1]);
        out[3] = bf16_hi(q.w[1]);
    } else {
#pragma unroll
        for (int k = 0; k < 4; ++k) out[k] = __uint_as_float(q.w[k]);
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) out[k] = v + k < hi ? fmaxf(out[k], nbig) : -INFINITY;
}

// Level-1 Gumbel score of a chunk: its log-sum-exp of l' plus its Gumbel variate (-inf for a chunk
// without mass).
// ln S with the hardware logarithm: S >= 1 for a chunk with mass (its maximum contributes 1), so the
// absolute error stays near 1e-6, far inside the near-tie allowance of the scores (1e-5 relative).
__device__ __forceinline__ float chunk_score(float m_raw, float S, float inv_tau, float gumbel) {
    return (m_raw * inv_tau + __logf(S)) + gumbel;
}

// Running statistics of a set of chunk records: the first chunk holding the raw maximum, the level-1
// winner (score, chunk), and S, T of the chunks with mass relative to the reference `ref`
// (S = sum exp(l' - ref), T = sum exp(l' - ref)(l' - ref)).
struct RowAcc {
    float mv, bs, ref, S, T;
    int jm, bj;
};
__device__ __forceinline__ void acc_init(RowAcc& a) {
    a.mv = a.bs = a.ref = -INFINITY;
    a.S = a.T = 0.f;
    a.jm = a.bj = 0x7fffffff;
}
// (S, T) of b folded into a: both rescaled to the larger reference.
__device__ __forceinline__ void acc_sums(RowAcc& a, float ref, float S, float T) {
    if (!(S > 0.f)) return;
    if (!(a.S > 0.f)) {
        a.ref = ref;
        a.S = S;
        a.T = T;
        return;
    }
    const float nr = fmaxf(a.ref, ref);
    const float da = a.ref - nr, db = ref - nr;
    const float ea = __expf(da), eb = __expf(db);
    a.T = fmaf(ea, fmaf(a.S, da, a.T), eb * fmaf(S, db, T));
    a.S = fmaf(a.S, ea, S * eb);
    a.ref = nr;
}
// b folded into a (both sets' statistics): larger value wins, equal values go to the smaller chunk.
__device__ __forceinline__ void acc_merge(RowAcc& a, const RowAcc& b) {
    if (b.mv > a.mv || (b.mv == a.mv && b.jm < a.jm)) {
        a.mv = b.mv;
        a.jm = b.jm;
    }
    if (b.bs > a.bs || (b.bs == a.bs && b.bj < a.bj)) {
        a.bs = b.bs;
        a.bj = b.bj;
    }
    acc_sums(a, b.ref, b.S, b.T);
}
__device__ __forceinline__ RowAcc acc_shfl_xor(const RowAcc& a, int o) {
    RowAcc b;
    b.mv = __shfl_xor_sync(0xffffffffu, a.mv, o);
    b.bs = __shfl_xor_sync(0xffffffffu, a.bs, o);
    b.ref = __shfl_xor_sync(0xffffffffu, a.ref, o);
    b.S = __shfl_xor_sync(0xffffffffu, a.S, o);
    b.T = __shfl_xor_sync(0xffffffffu, a.T, o);
    b.jm = __shfl_xor_sync(0xffffffffu, a.jm, o);
    b.bj = __shfl_xor_sync(0xffffffffu, a.bj, o);
    return b;
}

struct MergeShared {
    float f[2 * kPassWarps];
    int i[2 * kPassWarps];
    RowAcc acc[kPassWarps];
    int flag;
};

// Per-row merge, run by the merge kernel's CTA of the row.  Global memory is visited in two round trips:
// the chunk records (thread t holds quads of four consecutive chunks 4q .. 4q+3, q = t + u T, in
// registers, so one Philox call serves four chunk Gumbel variates), then the two chunks that must
// be re-read (the one holding the argmax and the level-1 winner), fetched together.
//
// Two block-wide exchanges: (1) the argmax over the chunk maxima, the level-1 winner and the
// log-sum-exp merge of (S, T) together (an online merge at a running reference), which fixes both
// chunks to re-read; (2) the argmax inside the argmax chunk and the level-2 winner.
// A re-read chunk is kQuads quads of four consecutive ids per thread: ids lo + 4 (tid + u T) + k.
constexpr int kQuads = kChunk / (4 * kPassThreads);
constexpr int kRecQuads = (512 / 4 + kPassThreads - 1) / kPassThreads;
static_assert(kQuads >= 1 && kChunk == 4 * kQuads * kPassThreads, "a chunk splits into whole quads per thread");

template <bool kBf16, int kKind>
__device__ __noinline__ void merge_row(const PassParams& p, int32_t row, int32_t canvas, float inv_tau,
                                       const void* rowp, MergeShared& sh) {
    const int tid = threadIdx.x;
    const int32_t nch = p.n_chunks;
    const unsigned long long* rec = p.rec + static_cast<size_t>(row) * nch * kRecWords;
    const unsigned tag = call_tag(p);
    const float nbig = neg_big(kBf16);
    const bool sampling = kKind == kPassSampler && p.mode != DG_X0_GREEDY;

    // The chunk Gumbel variates depend only on (seed, step, row, chunk): computed before the row's
    // records are ready, while its last streaming CTAs may still run.
    float gum[kRecQuads][4];
#pragma unroll
    for (int u = 0; u < kRecQuads; ++u) {
        const int32_t q = tid + u * kPassThreads;
        if (sampling && 4 * q < nch) {
            const uint4 w = philox4x32_10(
                make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(row), p.step, kDomChunkGumbel), p.key0,
                p.key1);
#pragma unroll
            for (int k = 0; k < 4; ++k) gum[u][k] = gumbel_from_word(word_of(w, k));
        } else {
#pragma unroll
            for (int k = 0; k < 4; ++k) gum[u][k] = 0.f;
        }
        // pin: computed here, before the wait, not where the scores are formed
        asm volatile("" ::"f"(gum[u][0]), "f"(gum[u][1]), "f"(gum[u][2]), "f"(gum[u][3]));
    }
    // Wait (bounded) until every record this thread will read carries this call's tag: the quads
    // q = tid + u T that stay in registers (rows up to 512 chunks) and the ones further out, which
    // are re-read from L2 in each pass below.  Every streaming CTA has started before this grid
    // launches, so the wait depends on no CTA still to be placed.
    float4 r[kRecQuads][4];
    {
        const long long limit = p.merge_wait_limit > 0 ? p.merge_wait_limit : kMergeWaitLimit;
        const long long t0 = clock64();
        bool ready = false;
        while (true) {
            ready = true;
#pragma unroll
            for (int u = 0; u < kRecQuads; ++u)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const int32_t j = 4 * (tid + u * kPassThreads) + k;
                    r[u][k] = j < nch ? get_record<kBf16>(rec, j, tag, ready) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
                }
            for (int32_t j = 4 * (tid + kRecQuads * kPassThreads); j < nch && ready; j += 4 * kPassThreads)
                for (int k = 0; k < 4 && j + k < nch; ++k) (void)get_record<kBf16>(rec, j + k, tag, ready);
            if (ready) break;
            if (clock64() - t0 > limit) {
                atomicMax(&g_pass_error, 1);
                break;
            }
            __nanosleep(64);
        }
    }
    __syncthreads();

    float target_logit = 0.f;
    bool target_ok = false;
    int32_t b_seq = 0, i_seq = 0;
    if (kKind == kPassCE && tid == 0) {
        b_seq = row / p.C;
        i_seq = row - b_seq * p.C;
        const int32_t k = p.canvas_idx[b_seq];
        DG_CHECK(g_pass_error, k >= 0 && k < p.K);  // a canvas index the caller gave
        if (k >= 0 && k < p.K) {
            const int32_t target =
                p.x0[static_cast<int64_t>(b_seq) * p.seq_len + p.P + static_cast<int64_t>(k) * p.C + i_seq];
            DG_CHECK(g_pass_error, target >= 0 && target < p.V);  // a token id the caller gave
            if (target >= 0 && target < p.V) {
                target_logit = load_logit(rowp, target, kBf16);
                target_ok = true;
            }
        }
    }

    // What thread 0 needs at the very end, fetched or computed while the records are in flight:
    // the current token, the canvas's Step thresholds and the Step's Philox words.
    int32_t xt = 0;
    unsigned long long thr_sd = 0, thr_jd = 0, thr_ss = 0;
    uint4 step_w = make_uint4(0u, 0u, 0u, 0u);
    // output pointers, read from the parameter bank now rather than after the last exchange
    int32_t* const out_x0 = p.x0_hat;
    int32_t* const out_am = p.argmax;
    float* const out_mp = p.max_prob;
    float* const out_lse = p.lse;
    float* const out_h = p.entropy;
    if (kKind == kPassSampler && tid == 0) asm volatile("" ::"l"(out_x0), "l"(out_am), "l"(out_mp), "l"(out_lse), "l"(out_h));
    if (kKind == kPassSampler && tid == 0 && p.x_next) {
        xt = p.x_t[row];
        DG_CHECK(g_pass_error, xt >= 0 && xt < p.V);  // a token id the caller gave
        thr_sd = p.thr_stay_diff[canvas];
        thr_jd = p.thr_jump_diff[canvas];
        thr_ss = p.thr_stay_same[canvas];
        step_w = philox4x32_10(make_uint4(0u, static_cast<uint32_t>(row), p.step, kDomStep), p.key0, p.key1);
        // pin the words here: computed while the records are in flight, not at the end
        asm volatile("" ::"r"(step_w.x), "r"(step_w.y), "l"(thr_sd), "l"(thr_jd), "l"(thr_ss), "r"(xt));
    }
    // Records beyond those (rows longer than 262144 ids) are re-read from L2 in each pass.
    constexpr int kFar = kRecQuads * kPassThreads;
    auto far_quad = [&](int32_t q, float4 (&f)[4]) {
        bool ok = true;  // checked above
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int32_t j = 4 * q + k;
            f[k] = j < nch ? get_record<kBf16>(rec, j, tag, ok) : make_float4(-INFINITY, 0.f, 0.f, 0.f);
        }
    };

    // (1) One block exchange for all of the row's statistics: each thread folds its records (the
    // first chunk holding the raw maximum, the level-1 winner of the chunk scores lse_c + G_c, and
    // (S, T) at a running reference), then the warps fold theirs by shuffles in a fixed tree and
    // every thread folds the warps' results in warp order (deterministic).
    RowAcc acc;
    acc_init(acc);
    auto fold = [&](int32_t j, const float4& f, float g) {
        if (j >= nch) return;
        if (f.x > acc.mv) {  // ascending chunks within a thread, strict: the first maximum wins
            acc.mv = f.x;
            acc.jm = j;
        }
        if (sampling) {
            const float sc = chunk_score(f.x, f.y, inv_tau, g);
            if (sc > acc.bs) {
                acc.bs = sc;
                acc.bj = j;
            }
        }
        acc_sums(acc, f.x * inv_tau, f.y, f.z);
    };
#pragma unroll
    for (int u = 0; u < kRecQuads; ++u)
#pragma unroll
        for (int k = 0; k < 4; ++k) fold(4 * (tid + u * kPassThreads) + k, r[u][k], gum[u][k]);
    for (int32_t q = tid + kFar; 4 * q < nch; q += kPassThreads) {
        float4 f[4];
        far_quad(q, f);
        float g[4] = {0.f, 0.f, 0.f, 0.f};
        if (sampling) {
            const uint4 w = philox4x32_10(
                make_uint4(static_cast<uint32_t>(q), static_cast<uint32_t>(row), p.step, kDomChunkGumbel), p.key0,
                p.key1);
#pragma unroll
            for (int k = 0; k < 4; ++k) g[k] = gumbel_from_word(word_of(w, k));
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) fold(4 * q + k, f[k], g[k]);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc_merge(acc, acc_shfl_xor(acc, o));
    if ((tid & 31) == 0) sh.acc[tid >> 5] = acc;
    __syncthreads();
    acc = sh.acc[0];
#pragma unroll
    for (int w = 1; w < kPassWarps; ++w) acc_merge(acc, sh.acc[w]);

    const float m_raw = acc.mv;
    int32_t jm = acc.jm, bj = acc.bj;
    DG_CHECK(g_pass_error, jm < nch);                                 // NaN logits only
    DG_CHECK(g_pass_error, !sampling || !(acc.S > 0.f) || bj < nch);  // likewise
    if (jm >= nch) jm = 0;  // only reachable with NaN inputs; keeps every index in range
    if (!sampling || bj >= nch) bj = jm;  // greedy, or NaN scores only
    const float m_row = m_raw * inv_tau;
    // (S, T) at the row maximum (the reference is the maximum unless the maximum chunk is masked)
    float S = acc.S, T = acc.T;
    if (S > 0.f && acc.ref != m_row) {
        const float d = acc.ref - m_row;
        const float e = __expf(d);
        T = e * fmaf(S, d, T);
        S *= e;
    }

    // Both re-read chunks are known: quads of ids lo + 4 (tid + u T) .. + 3 of each, loaded now as
    // raw words, with the level-2 chunk's Philox words computed while the loads are in flight.
    const int32_t alo = jm * kChunk, ahi = min(alo + kChunk, p.V);
    const int32_t glo = bj * kChunk, ghi = min(glo + kChunk, p.V);
    RawQuad araw[kQuads], graw[kQuads];
    uint4 tw[kQuads];
    if (kKind == kPassSampler) {
#pragma unroll
        for (int u = 0; u < kQuads; ++u) {
            const int32_t o = 4 * (tid + u * kPassThreads);
            araw[u] = load_quad<kBf16>(rowp, alo + o, ahi);
            graw[u] = load_quad<kBf16>(rowp, glo + o, ghi);
        }
#pragma unroll
        for (int u = 0; u < kQuads; ++u) {
            const int32_t vg0 = glo + 4 * (tid + u * kPassThreads);
            tw[u] = sampling ? philox4x32_10(make_uint4(static_cast<uint32_t>(vg0) >> 2, static_cast<uint32_t>(row),
                                                        p.step, kDomTokenGumbel),
                                             p.key0, p.key1)
                             : make_uint4(0u, 0u, 0u, 0u);
        }
    }
    const float ln_s = logf(S);
    const float lse = m_row + ln_s;

    if (kKind == kPassStats) {
        if (tid == 0) {
            p.lse[row] = lse;
        }
        return;
    }

    if (kKind == kPassCE) {
        if (tid == 0) {
            const float loss = target_ok ? lse - target_logit : __int_as_float(0x7fc00000);  // NaN: bad target
            p.loss_rows[row] = loss;
            if (p.lse) p.lse[row] = lse;
            __threadfence();
            const unsigned prev = atomicAdd(&p.seq_ticket[b_seq], 1u);
            const bool last = prev == static_cast<unsigned>(p.C - 1);
            if (last) __threadfence();
            sh.flag = last;
            sh.i[0] = b_seq;
        }
        __syncthreads();
        if (!sh.flag) return;
        const int32_t b = sh.i[0];
        float acc = 0.f;
        for (int32_t q = tid; q < p.C; q += kPassThreads) acc += ld_cg_f(p.loss_rows + static_cast<int64_t>(b) * p.C + q);
        const float total = block_sum<kPassWarps>(acc, sh.f);
        if (tid == 0) {
            if (p.loss_seq) p.loss_seq[b] = total;
            p.seq_ticket[b] = 0u;
        }
        return;
    }

    // ---- sampler epilogue
    // (2) The first id of the argmax chunk holding the row maximum, and the level-2 winner
    // argmax of l'_v + G_v over the level-1 chunk (four ids per Philox call).
    float av[kQuads][4], gv[kQuads][4];
#pragma unroll
    for (int u = 0; u < kQuads; ++u) {
        const int32_t o = 4 * (tid + u * kPassThreads);
        unpack_quad<kBf16>(araw[u], alo + o, ahi, nbig, av[u]);
        unpack_quad<kBf16>(graw[u], glo + o, ghi, nbig, gv[u]);
    }
    float amv = -INFINITY;
    int am = 0x7fffffff;
#pragma unroll
    for (int u = 0; u < kQuads; ++u)  // ascending ids, strict: the first maximum wins
#pragma unroll
        for (int k = 0; k < 4; ++k)
            if (av[u][k] > amv) {
                amv = av[u][k];
                am = alo + 4 * (tid + u * kPassThreads) + k;
            }
    float bs2 = -INFINITY;
    int bv = 0x7fffffff;
#pragma unroll
    for (int u = 0; u < kQuads; ++u) {
        const int32_t vg0 = glo + 4 * (tid + u * kPassThreads);
        if (sampling && vg0 < ghi) {
            const uint4 w = tw[u];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                if (vg0 + k < ghi) {
                    const float sc = gv[u][k] * inv_tau + gumbel_from_word(word_of(w, k));
                    if (sc > bs2) {
                        bs2 = sc;
                        bv = vg0 + k;
                    }
                }
            }
        }
    }
    block_argmax2<kPassWarps>(amv, am, bs2, bv, sh.f, sh.i);
    DG_CHECK(g_pass_error, am >= alo && am < ahi);  // NaN logits only
    if (am < alo || am >= ahi) am = alo;
    const int32_t x0 = sampling && bv >= glo && bv < ghi ? bv : am;

    if (tid == 0) {
        if (p.x_next) {  // the Step posterior (skipped when a per-canvas rule decides instead)
            unsigned long long t_stay, t_jump;
            if (x0 != xt) {
                t_stay = thr_sd;
                t_jump = thr_jd;
            } else {
                t_stay = thr_ss;
                t_jump = t_stay;
            }
            const uint4 w = step_w;
            const unsigned long long u = w.x;
            int32_t xn;
            uint8_t br;
            if (u < t_stay) {
                xn = xt;
                br = 0;
            } else if (u < t_jump) {
                xn = x0;
                br = 1;
            } else {
                xn = word_to_index(w.y, p.V);
                br = 2;
            }
            if (DG_CHECKED(g_pass_error, xn >= 0 && xn < p.V)) p.x_next[row] = xn;
            if (p.branch) p.branch[row] = br;
        }
        if (out_x0 && DG_CHECKED(g_pass_error, (x0 >= alo && x0 < ahi) || (x0 >= glo && x0 < ghi))) out_x0[row] = x0;
        if (out_am && DG_CHECKED(g_pass_error, am >= 0 && am < p.V)) out_am[row] = am;
        if (out_mp) out_mp[row] = 1.0f / S;
        if (out_lse) out_lse[row] = lse;
        if (out_h) out_h[row] = ln_s - T / S;
    }
}

template <bool kBf16, int kKind>
__global__ void __launch_bounds__(kPassThreads, kBf16 ? 10 : 4) logits_pass_kernel(const __grid_constant__ PassParams p) {
    // The merge kernel, launched as a programmatic dependent, may start once every CTA of this grid
    // has started; each merge waits only for its own row's records.
    if (threadIdx.x == 0) grid_launch_dependents();
    const int32_t row = blockIdx.x / p.segs;
    const int32_t seg = blockIdx.x - row * p.segs;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int32_t canvas = row / p.C;
    const float inv_tau = kKind == kPassCE ? 1.0f : p.inv_tau[canvas];
    constexpr int kElt = kBf16 ? 2 : 4;
    const char* rowp = reinterpret_cast<const char*>(p.logits) + static_cast<size_t>(row) * p.ld * kElt;
    unsigned long long* rec = p.rec + static_cast<size_t>(row) * p.n_chunks * kRecWords;
    const unsigned tag = call_tag(p);

    // Groups of 4 chunks (2048 ids) per warp-iteration; this CTA owns groups [g_begin, g_end).
    const int32_t n_groups = (p.V + 4 * kChunk - 1) / (4 * kChunk);
    const int32_t g_begin = seg * p.groups_per_cta;
    const int32_t g_end = min(g_begin + p.groups_per_cta, n_groups);
    for (int32_t gi = g_begin + warp; gi < g_end; gi += kPassWarps) {
        const int32_t lo = gi * 4 * kChunk;
        ChunkStats cs;
        if (lo + 4 * kChunk <= p.V)
            cs = kBf16 ? group_full_bf16(rowp + static_cast<size_t>(lo) * kElt, lane, inv_tau)
                       : group_full_f32(rowp + static_cast<size_t>(lo) * kElt, lane, inv_tau);
        else
            cs = group_ragged(rowp, kBf16, lo, p.V, lane, inv_tau);
        const int32_t c = 4 * gi + (lane >> 3);
        if ((lane & 7) == 0 && c < p.n_chunks)
            put_record<kBf16>(rec + static_cast<size_t>(c) * kRecWords, cs.m_raw, cs.S, cs.T, tag);
    }
}

// Per-row merge of the chunk records: one CTA per row, launched as a programmatic dependent of the
// streaming kernel.  Its own dependents (a contraction reading lse) may start as soon as every
// merge CTA has started; they wait for the merges to finish.
template <bool kBf16, int kKind>
__global__ void __launch_bounds__(kPassThreads) merge_kernel(const __grid_constant__ PassParams p) {
    __shared__ MergeShared sh;
    if (threadIdx.x == 0) grid_launch_dependents();
    const int32_t row = blockIdx.x;
    const int32_t canvas = row / p.C;
    const float inv_tau = kKind == kPassCE ? 1.0f : p.inv_tau[canvas];
    constexpr int kElt = kBf16 ? 2 : 4;
    const char* rowp = reinterpret_cast<const char*>(p.logits) + static_cast<size_t>(row) * p.ld * kElt;
    merge_row<kBf16, kKind>(p, row, canvas, inv_tau, rowp, sh);
    // The last merge CTA advances the call counter: every CTA of this call has read it by then, and
    // the next call's kernels start after this grid ends.
    if (threadIdx.x == 0 && atomicAdd(&p.epoch[1], 1u) == gridDim.x - 1) {
        p.epoch[1] = 0u;
        p.epoch[0] += 1u;
    }
}

}  // namespace

cudaError_t launch_logits_pass(const PassParams& p, int kind, int is_bf16, cudaStream_t s) {
    const long long grid = static_cast<long long>(p.R) * p.segs;
    if (grid <= 0 || grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
    if (p.groups_per_cta != kPassWarps) return cudaErrorInvalidValue;  // the kernel maps one group per warp
    const dim3 g(static_cast<unsigned>(grid)), b(kPassThreads);
    // the merge: one CTA per row, a programmatic dependent of the streaming kernel
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(static_cast<unsigned>(p.R));
    cfg.blockDim = b;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    cudaError_t e = cudaSuccess;
#define DG_LAUNCH(BF, K)                                                  \
    do {                                                                  \
        logits_pass_kernel<BF, K><<<g, b, 0, s>>>(p);                     \
        e = cudaGetLastError();                                           \
        if (e == cudaSuccess) e = cudaLaunchKernelEx(&cfg, merge_kernel<BF, K>, p); \
    } while (0)
    if (is_bf16) {
        if (kind == kPassSampler) DG_LAUNCH(true, kPassSampler);
        else if (kind == kPassStats) DG_LAUNCH(true, kPassStats);
        else DG_LAUNCH(true, kPassCE);
    } else {
        if (kind == kPassSampler) DG_LAUNCH(false, kPassSampler);
        else if (kind == kPassStats) DG_LAUNCH(false, kPassStats);
        else DG_LAUNCH(false, kPassCE);
    }
#undef DG_LAUNCH
    note_launches(2);
    return e;
}

cudaError_t launch_merge_only(const PassParams& p, int is_bf16, cudaStream_t s) {
    if (p.R < 1) return cudaErrorInvalidConfiguration;
    if (is_bf16) merge_kernel<true, kPassStats><<<p.R, kPassThreads, 0, s>>>(p);
    else merge_kernel<false, kPassStats><<<p.R, kPassThreads, 0, s>>>(p);
    note_launches(1);
    return cudaGetLastError();
}

cudaError_t read_and_clear_pass_error(int* out) {
    int v = 0;
    cudaError_t e = cudaMemcpyFromSymbol(&v, g_pass_error, sizeof(int));
    if (e != cudaSuccess) return e;
    if (v) {
        const int zero = 0;
        e = cudaMemcpyToSymbol(g_pass_error, &zero, sizeof(int));
    }
    *out = v;
    return e;
}

}  // namespace dg
