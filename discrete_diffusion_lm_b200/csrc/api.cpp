// Host side of the C ABI declared in include/dg.h: argument checks, per-canvas thresholds in
// double, workspace layout, launches on the caller's stream.  No device memory is allocated here.
#include <cuda_runtime.h>

#include <atomic>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <string>

#include "../../include/dg.h"
#include "../../include/dg_test.h"
#include "kernels.cuh"

namespace dg {

namespace {

thread_local std::string g_last_error;
std::atomic<uint64_t> g_launches{0};

int fail(int code, const char* fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    std::vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    g_last_error = buf;
    return code;
}

int cuda_fail(cudaError_t e, const char* what) {
    return fail(DG_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

// The kernels are built for sm_100a only; refuse any other device up front.
int check_device() {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
    static std::atomic<int> known[64];
    if (dev >= 0 && dev < 64) {
        const int k = known[dev].load();
        if (k == 1) return DG_OK;
        if (k == 2) return fail(DG_ERR_UNSUPPORTED, "device %d is not compute capability 10.0 (sm_100a)", dev);
    }
    int major = 0, minor = 0;
    e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    const bool ok = major == 10 && minor == 0;
    if (dev >= 0 && dev < 64) known[dev].store(ok ? 1 : 2);
    if (!ok) return fail(DG_ERR_UNSUPPORTED, "device %d is sm_%d%d; this library is built for sm_100a", dev, major, minor);
    return DG_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Noise schedule kappa_t: linear 1 - t or cosine cos^2(pi t / 2), in double.
double kappa(int schedule, double t) {
    if (schedule == DG_SCHED_LINEAR) return 1.0 - t;
    const double c = std::cos(M_PI * t / 2.0);
    return c * c;
}

// Integer threshold T with (w < T) <=> (w 2^-32 < x) for every 32-bit w: T = ceil(x 2^32),
// clamped to [0, 2^32].  x 2^32 is exact in double, so the comparison is the exact one.
unsigned long long prob_threshold(double x) {
    if (!(x > 0.0)) return 0ull;
    if (x >= 1.0) return 1ull << 32;
    return static_cast<unsigned long long>(std::ceil(x * 4294967296.0));
}

// Step thresholds of one canvas: the exact posterior of the uniform mixture path,
// P(X_s | X_t = a, X_0 = b) with alpha = kappa_t / kappa_s, as a three-way mixture of
// "stay at a", "jump to b" and "uniform over V":
//   b != a: stay = alpha (1 - kappa_s) / (1 - kappa_t), jump = (1 - alpha) kappa_s / (1 - kappa_t)
//   b == a: uniform = (1 - alpha)(1 - kappa_s) / (V (kappa_t + (1 - kappa_t)/V)), stay = 1 - uniform
// If kappa_s <= kappa_t (dt = 0 in effect) the state stays: every threshold is 2^32.
void step_thresholds(int schedule, double t, double dt, int32_t V, unsigned long long* stay_diff,
                     unsigned long long* jump_diff, unsigned long long* stay_same) {
    double s = t - dt;
    if (s < 0.0) s = 0.0;
    const double kt = kappa(schedule, t), ks = kappa(schedule, s);
    if (ks <= kt) {
        *stay_diff = *jump_diff = *stay_same = 1ull << 32;
        return;
    }
    const double alpha = kt / ks;
    const double stay = alpha * (1.0 - ks) / (1.0 - kt);
    const double jump = (1.0 - alpha) * ks / (1.0 - kt);
    *stay_diff = prob_threshold(stay);
    *jump_diff = prob_threshold(stay + jump);
    const double D = kt + (1.0 - kt) / static_cast<double>(V);
    const double uniform = (1.0 - alpha) * (1.0 - ks) / (static_cast<double>(V) * D);
    *stay_same = prob_threshold(1.0 - uniform);
}

// Threshold for sums of fixed-point entropies q = floor(H 2^32): (sum q < T) <=> (sum q < x 2^32),
// T = ceil(x 2^32) (x 2^32 is exact in double), clamped to [0, 2^63).
long long entropy_threshold(double x) {
    if (!(x > 0.0)) return 0;
    const double y = std::ceil(x * 4294967296.0);
    if (y >= 9.0e18) return 0x7fffffffffffffffLL;
    return static_cast<long long>(y);
}

int32_t n_chunks_of(int32_t V) { return (V + kChunk - 1) / kChunk; }

// Groups of 4 chunks (2048 ids) per CTA of the logits pass: one per warp.
int32_t n_groups_of(int32_t V) { return (V + 4 * kChunk - 1) / (4 * kChunk); }
int32_t groups_per_cta_of(int32_t /*n_groups*/) { return kPassWarps; }

// Logits-pass workspace: the call counter and merge ticket, sequence tickets (canvas CE), then the
// tagged chunk records.
struct PassWs {
    unsigned* epoch;
    uint32_t* seq_ticket;
    unsigned long long* rec;
};
size_t pass_ws_bytes(int32_t R, int32_t V, int32_t n_seq) {
    return 256 + align_up(static_cast<size_t>(n_seq) * 4, 256) +
           static_cast<size_t>(R) * n_chunks_of(V) * kRecWords * 8;
}
PassWs carve_pass_ws(void* ws, int32_t /*R*/, int32_t n_seq) {
    char* p = static_cast<char*>(ws);
    PassWs w;
    w.epoch = reinterpret_cast<unsigned*>(p);
    p += 256;
    w.seq_ticket = reinterpret_cast<uint32_t*>(p);
    p += align_up(static_cast<size_t>(n_seq) * 4, 256);
    w.rec = reinterpret_cast<unsigned long long*>(p);
    return w;
}

bool valid_dtype(int d) { return d == DG_F32 || d == DG_BF16; }
int elt_size(int d) { return d == DG_BF16 ? 2 : 4; }

int check_logits(const void* logits, int dtype, int64_t ld, int32_t V) {
    if (!logits) return fail(DG_ERR_INVALID_ARG, "logits is NULL");
    if (!valid_dtype(dtype)) return fail(DG_ERR_INVALID_ARG, "logits dtype %d is not DG_F32 or DG_BF16", dtype);
    if (V < 1) return fail(DG_ERR_INVALID_ARG, "V = %d must be >= 1", V);
    if (V > DG_MAX_VOCAB) return fail(DG_ERR_INVALID_ARG, "V = %d exceeds DG_MAX_VOCAB = %d", V, DG_MAX_VOCAB);
    if (ld < V) return fail(DG_ERR_INVALID_ARG, "ld = %lld is smaller than V = %d", (long long)ld, V);
    if (!aligned16(logits)) return fail(DG_ERR_ALIGNMENT, "logits base is not 16-byte aligned");
    if ((ld * elt_size(dtype)) % 16 != 0)
        return fail(DG_ERR_ALIGNMENT, "ld * element size = %lld bytes is not a multiple of 16",
                    (long long)(ld * elt_size(dtype)));
    return DG_OK;
}

int check_canvases(int32_t B, int32_t C) {
    if (B < 1 || B > DG_MAX_CANVASES) return fail(DG_ERR_INVALID_ARG, "B = %d must be in [1, %d]", B, DG_MAX_CANVASES);
    if (C < 1) return fail(DG_ERR_INVALID_ARG, "C = %d must be >= 1", C);
    if (static_cast<long long>(B) * C > 0x7fffffffLL) return fail(DG_ERR_INVALID_ARG, "B * C overflows int32");
    return DG_OK;
}

int check_inv_tau(const float* inv_tau, int32_t B, float* out) {
    for (int32_t b = 0; b < B; ++b) {
        const float v = inv_tau ? inv_tau[b] : 1.0f;
        if (!(v > 0.0f) || !(v <= 1.0e6f))
            return fail(DG_ERR_INVALID_ARG, "inv_tau[%d] = %g must be in (0, 1e6]", b, static_cast<double>(v));
        out[b] = v;
    }
    return DG_OK;
}

}  // namespace

void note_launches(uint64_t n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

void set_error_message(int /*code*/, const char* msg) { g_last_error = msg ? msg : ""; }

}  // namespace dg

using namespace dg;

extern "C" {

const char* dg_last_error(void) { return g_last_error.c_str(); }

const char* dg_version(void) { return "dg 0.1 (sm_100a)"; }

uint64_t dg_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

int dg_device_error(int* code) {
    g_last_error.clear();
    if (!code) return fail(DG_ERR_INVALID_ARG, "code is NULL");
    int rc;
    if ((rc = check_device()) != DG_OK) return rc;
    const cudaError_t e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
    int c[4] = {0, 0, 0, 0};
    cudaError_t r = read_and_clear_device_error(&c[0]);
    if (r == cudaSuccess) r = read_and_clear_pass_error(&c[1]);
    if (r == cudaSuccess) r = read_and_clear_ops_error(&c[2]);
    if (r == cudaSuccess) r = read_and_clear_noise_error(&c[3]);
    if (r != cudaSuccess) return cuda_fail(r, "reading the device error words");
    *code = 0;
    for (int k = 0; k < 4; ++k)  // the largest code: a failed check (2) before an expired wait (1)
        if (c[k] > *code) *code = c[k];
    return DG_OK;
}

size_t dg_sampler_step_workspace_size(int32_t rows, int32_t V) {
    if (rows < 1 || V < 1) return 0;
    return pass_ws_bytes(rows, V, 0);
}

int dg_sampler_step(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t, int32_t B, int32_t C,
                    int32_t V, int schedule, const double* t, const double* dt, const float* inv_tau, uint64_t seed,
                    uint32_t step, int x0_mode, int32_t* x_next, int32_t* x0_hat, int32_t* argmax, float* max_prob,
                    float* lse, float* entropy, uint8_t* branch, void* workspace, size_t workspace_bytes,
                    dg_stream_t stream) {
    return dg::sampler_step_impl(logits, logits_dtype, ld, x_t, B, C, V, schedule, t, dt, inv_tau, seed, step, x0_mode,
                                 x_next, x0_hat, argmax, max_prob, lse, entropy, branch, workspace, workspace_bytes,
                                 stream, false);
}

}  // extern "C"

namespace dg {

// The sampler step behind dg_sampler_step and dg_sampler_step_noalloc.  Every argument is checked
// before anything is enqueued; with clear_ws the workspace is zeroed on the stream (after the
// checks, right before the launches).
int sampler_step_impl(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t, int32_t B, int32_t C,
                      int32_t V, int schedule, const double* t, const double* dt, const float* inv_tau, uint64_t seed,
                      uint32_t step, int x0_mode, int32_t* x_next, int32_t* x0_hat, int32_t* argmax, float* max_prob,
                      float* lse, float* entropy, uint8_t* branch, void* workspace, size_t workspace_bytes,
                      dg_stream_t stream, bool clear_ws) {
    g_last_error.clear();
    int rc;
    if ((rc = check_logits(logits, logits_dtype, ld, V)) != DG_OK) return rc;
    if ((rc = check_canvases(B, C)) != DG_OK) return rc;
    if (!x_t || !x_next) return fail(DG_ERR_INVALID_ARG, "x_t and x_next are required");
    if (!t || !dt) return fail(DG_ERR_INVALID_ARG, "t and dt (host arrays) are required");
    if (schedule != DG_SCHED_LINEAR && schedule != DG_SCHED_COSINE)
        return fail(DG_ERR_INVALID_ARG, "schedule %d is not LINEAR or COSINE", schedule);
    if (x0_mode != DG_X0_SAMPLE && x0_mode != DG_X0_GREEDY)
        return fail(DG_ERR_INVALID_ARG, "x0_mode %d is not SAMPLE or GREEDY", x0_mode);
    const int32_t R = B * C;
    const size_t need = pass_ws_bytes(R, V, 0);
    if (!workspace || workspace_bytes < need)
        return fail(DG_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
    if (!aligned16(workspace)) return fail(DG_ERR_ALIGNMENT, "workspace is not 16-byte aligned");

    static thread_local PassParams p;
    std::memset(&p, 0, sizeof(p));
    if ((rc = check_inv_tau(inv_tau, B, p.inv_tau)) != DG_OK) return rc;
    for (int32_t b = 0; b < B; ++b) {
        if (!(t[b] >= 0.0 && t[b] <= 1.0)) return fail(DG_ERR_INVALID_ARG, "t[%d] = %g is outside [0, 1]", b, t[b]);
        if (!(dt[b] >= 0.0) || !std::isfinite(dt[b]))
            return fail(DG_ERR_INVALID_ARG, "dt[%d] = %g must be finite and >= 0", b, dt[b]);
        step_thresholds(schedule, t[b], dt[b], V, &p.thr_stay_diff[b], &p.thr_jump_diff[b], &p.thr_stay_same[b]);
    }
    if ((rc = check_device()) != DG_OK) return rc;

    const PassWs w = carve_pass_ws(workspace, R, 0);
    p.logits = logits;
    p.ld = ld;
    p.R = R;
    p.C = C;
    p.V = V;
    p.n_chunks = n_chunks_of(V);
    p.groups_per_cta = groups_per_cta_of(n_groups_of(V));
    p.segs = (n_groups_of(V) + p.groups_per_cta - 1) / p.groups_per_cta;
    p.rec = w.rec;
    p.epoch = w.epoch;
    p.x_t = x_t;
    p.key0 = static_cast<uint32_t>(seed);
    p.key1 = static_cast<uint32_t>(seed >> 32);
    p.step = step;
    p.mode = x0_mode;
    p.x_next = x_next;
    p.x0_hat = x0_hat;
    p.argmax = argmax;
    p.max_prob = max_prob;
    p.lse = lse;
    p.entropy = entropy;
    p.branch = branch;
    if (clear_ws) {
        const cudaError_t z = cudaMemsetAsync(workspace, 0, need, reinterpret_cast<cudaStream_t>(stream));
        if (z != cudaSuccess) return cuda_fail(z, "workspace clear");
    }
    const cudaError_t e = launch_logits_pass(p, kPassSampler, logits_dtype == DG_BF16, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "logits pass launch");
    return DG_OK;
}

}  // namespace dg

extern "C" {

int dg_forward_noise(const int32_t* x0, int32_t n_seq, int32_t P, int32_t K, int32_t C, int32_t V, int schedule,
                     const double* t, uint64_t seed, int32_t* x_t, int32_t* canvas_idx, dg_stream_t stream) {
    g_last_error.clear();
    if (!x0 || !x_t) return fail(DG_ERR_INVALID_ARG, "x0 and x_t are required");
    if (x0 == x_t) return fail(DG_ERR_INVALID_ARG, "x_t may not alias x0");
    if (!t) return fail(DG_ERR_INVALID_ARG, "t (host array) is required");
    if (n_seq < 1 || n_seq > DG_MAX_CANVASES)
        return fail(DG_ERR_INVALID_ARG, "n_seq = %d must be in [1, %d]", n_seq, DG_MAX_CANVASES);
    if (P < 0 || K < 1 || C < 1 || V < 1) return fail(DG_ERR_INVALID_ARG, "need P >= 0, K >= 1, C >= 1, V >= 1");
    const long long L = static_cast<long long>(P) + static_cast<long long>(K) * C;
    if (L > 0x7fffffffLL) return fail(DG_ERR_INVALID_ARG, "P + K*C overflows int32");
    if (schedule != DG_SCHED_LINEAR && schedule != DG_SCHED_COSINE)
        return fail(DG_ERR_INVALID_ARG, "schedule %d is not LINEAR or COSINE", schedule);
    static thread_local NoiseParams p;
    std::memset(&p, 0, sizeof(p));
    for (int32_t b = 0; b < n_seq; ++b) {
        if (!(t[b] >= 0.0 && t[b] <= 1.0)) return fail(DG_ERR_INVALID_ARG, "t[%d] = %g is outside [0, 1]", b, t[b]);
        p.keep_thr[b] = prob_threshold(kappa(schedule, t[b]));
    }
    int rc;
    if ((rc = check_device()) != DG_OK) return rc;
    p.x0 = x0;
    p.x_t = x_t;
    p.canvas_idx = canvas_idx;
    p.n_seq = n_seq;
    p.P = P;
    p.K = K;
    p.C = C;
    p.V = V;
    p.seq_len = L;
    p.key0 = static_cast<uint32_t>(seed);
    p.key1 = static_cast<uint32_t>(seed >> 32);
    const cudaError_t e = launch_forward_noise(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "forward noise launch");
    return DG_OK;
}

size_t dg_canvas_ce_workspace_size(int32_t n_seq, int32_t C, int32_t V) {
    if (n_seq < 1 || C < 1 || V < 1) return 0;
    return pass_ws_bytes(n_seq * C, V, n_seq);
}

int dg_canvas_ce(const void* logits, int logits_dtype, int64_t ld, const int32_t* x0, const int32_t* canvas_idx,
                 int32_t n_seq, int32_t P, int32_t K, int32_t C, int32_t V, float* loss_rows, float* loss_seq,
                 float* lse_rows, void* workspace, size_t workspace_bytes, dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if ((rc = check_logits(logits, logits_dtype, ld, V)) != DG_OK) return rc;
    if ((rc = check_canvases(n_seq, C)) != DG_OK) return rc;
    if (!x0 || !canvas_idx || !loss_rows) return fail(DG_ERR_INVALID_ARG, "x0, canvas_idx and loss_rows are required");
    if (P < 0 || K < 1) return fail(DG_ERR_INVALID_ARG, "need P >= 0 and K >= 1");
    if (static_cast<long long>(P) + static_cast<long long>(K) * C > 0x7fffffffLL)
        return fail(DG_ERR_INVALID_ARG, "P + K*C overflows int32");
    const int32_t R = n_seq * C;
    const size_t need = pass_ws_bytes(R, V, n_seq);
    if (!workspace || workspace_bytes < need)
        return fail(DG_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
    if (!aligned16(workspace)) return fail(DG_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
    if ((rc = check_device()) != DG_OK) return rc;
    static thread_local PassParams p;
    std::memset(&p, 0, sizeof(p));
    const PassWs w = carve_pass_ws(workspace, R, n_seq);
    p.logits = logits;
    p.ld = ld;
    p.R = R;
    p.C = C;
    p.V = V;
    p.n_chunks = n_chunks_of(V);
    p.groups_per_cta = groups_per_cta_of(n_groups_of(V));
    p.segs = (n_groups_of(V) + p.groups_per_cta - 1) / p.groups_per_cta;
    p.rec = w.rec;
    p.epoch = w.epoch;
    p.seq_ticket = w.seq_ticket;
    p.x0 = x0;
    p.canvas_idx = canvas_idx;
    p.P = P;
    p.K = K;
    p.seq_len = static_cast<int64_t>(P) + static_cast<int64_t>(K) * C;
    p.loss_rows = loss_rows;
    p.loss_seq = loss_seq;
    p.lse = lse_rows;
    for (int32_t b = 0; b < n_seq; ++b) p.inv_tau[b] = 1.0f;
    const cudaError_t e = launch_logits_pass(p, kPassCE, logits_dtype == DG_BF16, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "canvas CE launch");
    return DG_OK;
}

size_t dg_selfcond_workspace_size(int32_t rows, int32_t V, int32_t d, int logits_dtype, int embed_dtype,
                                  int have_lse) {
    if (rows < 1 || V < 1 || d < 1 || !valid_dtype(logits_dtype) || !valid_dtype(embed_dtype)) return 0;
    size_t n = 0;
    if (!have_lse) n += align_up(static_cast<size_t>(rows) * 4, 256) + align_up(pass_ws_bytes(rows, V, 0), 256);
    if (embed_dtype == DG_F32) n += align_up(static_cast<size_t>(V) * d * 2, 256);
    n += selfcond_partial_bytes(rows, V, d, logits_dtype == DG_BF16);
    return n;
}

}  // extern "C"

namespace {
int selfcond_impl(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C, int32_t V,
                  const float* inv_tau, const float* lse, const void* E, int embed_dtype, int32_t d, void* z,
                  void* workspace, size_t workspace_bytes, dg_stream_t stream, int32_t fault_block,
                  long long wait_limit, bool dependent = false, bool validate_only = false) {
    g_last_error.clear();
    int rc;
    if ((rc = check_logits(logits, logits_dtype, ld, V)) != DG_OK) return rc;
    if ((rc = check_canvases(B, C)) != DG_OK) return rc;
    if (!E || !z) return fail(DG_ERR_INVALID_ARG, "E and z are required");
    if (!valid_dtype(embed_dtype)) return fail(DG_ERR_INVALID_ARG, "E dtype %d is not DG_F32 or DG_BF16", embed_dtype);
    if (d < 64 || d > 16384 || d % 64 != 0)
        return fail(DG_ERR_INVALID_ARG, "d = %d must be a multiple of 64 in [64, 16384]", d);
    if (!aligned16(E) || !aligned16(z)) return fail(DG_ERR_ALIGNMENT, "E and z must be 16-byte aligned");
    if (lse && (reinterpret_cast<uintptr_t>(lse) & 3u)) return fail(DG_ERR_ALIGNMENT, "lse must be 4-byte aligned");
    const int32_t R = B * C;
    const size_t need = dg_selfcond_workspace_size(R, V, d, logits_dtype, embed_dtype, lse != nullptr);
    if (!workspace || workspace_bytes < need)
        return fail(DG_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
    if (!aligned16(workspace) || (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(DG_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    static thread_local SelfcondParams sp;
    std::memset(&sp, 0, sizeof(sp));
    if ((rc = check_inv_tau(inv_tau, B, sp.inv_tau)) != DG_OK) return rc;
    if (validate_only) return DG_OK;
    if ((rc = check_device()) != DG_OK) return rc;

    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    char* wp = static_cast<char*>(workspace);
    const float* lse_use = lse;
    if (!lse) {
        float* lse_ws = reinterpret_cast<float*>(wp);
        wp += align_up(static_cast<size_t>(R) * 4, 256);
        static thread_local PassParams p;
        std::memset(&p, 0, sizeof(p));
        const PassWs w = carve_pass_ws(wp, R, 0);
        wp += align_up(pass_ws_bytes(R, V, 0), 256);
        p.logits = logits;
        p.ld = ld;
        p.R = R;
        p.C = C;
        p.V = V;
        p.n_chunks = n_chunks_of(V);
        p.groups_per_cta = groups_per_cta_of(n_groups_of(V));
        p.segs = (n_groups_of(V) + p.groups_per_cta - 1) / p.groups_per_cta;
        p.rec = w.rec;
        p.epoch = w.epoch;
        p.lse = lse_ws;
        std::memcpy(p.inv_tau, sp.inv_tau, sizeof(float) * B);
        const cudaError_t e = launch_logits_pass(p, kPassStats, logits_dtype == DG_BF16, s);
        if (e != cudaSuccess) return cuda_fail(e, "statistics pass launch");
        lse_use = lse_ws;
    }
    const uint16_t* E16 = static_cast<const uint16_t*>(E);
    if (embed_dtype == DG_F32) {
        uint16_t* e16 = reinterpret_cast<uint16_t*>(wp);
        wp += align_up(static_cast<size_t>(V) * d * 2, 256);
        const cudaError_t e = launch_convert_f32_bf16(static_cast<const float*>(E), e16, static_cast<int64_t>(V) * d, s);
        if (e != cudaSuccess) return cuda_fail(e, "embedding conversion launch");
        E16 = e16;
    }
    sp.logits = logits;
    sp.ld = ld;
    sp.logits_bf16 = logits_dtype == DG_BF16;
    sp.lse = lse_use;
    sp.E = E16;
    sp.z = static_cast<uint16_t*>(z);
    sp.R = R;
    sp.C = C;
    sp.V = V;
    sp.d = d;
    // the partial sums live at the end of the workspace
    sp.partial = reinterpret_cast<float*>(wp);
    sp.wait_limit = wait_limit;
    sp.fault_block = fault_block;
    sp.dependent = dependent && lse != nullptr;
    const cudaError_t e = launch_selfcond(sp, s);
    if (e != cudaSuccess) return cuda_fail(e, "self-conditioning launch");
    return DG_OK;
}
}  // namespace

extern "C" {

int dg_selfcond(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C, int32_t V,
                const float* inv_tau, const float* lse, const void* E, int embed_dtype, int32_t d, void* z,
                void* workspace, size_t workspace_bytes, dg_stream_t stream) {
    return selfcond_impl(logits, logits_dtype, ld, B, C, V, inv_tau, lse, E, embed_dtype, d, z, workspace,
                         workspace_bytes, stream, -1, 0);
}

int dg_test_bounded_wait(uint32_t limit_cycles, dg_stream_t stream) {
    g_last_error.clear();
    if (limit_cycles == 0) return fail(DG_ERR_INVALID_ARG, "limit_cycles must be > 0");
    int rc;
    if ((rc = check_device()) != DG_OK) return rc;
    const cudaError_t e = launch_bounded_wait_test(static_cast<long long>(limit_cycles),
                                                   reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "bounded-wait test launch");
    return DG_OK;
}

int dg_test_selfcond_stall(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C, int32_t V,
                           const float* inv_tau, const float* lse, const void* E, int embed_dtype, int32_t d,
                           void* z, void* workspace, size_t workspace_bytes, dg_stream_t stream,
                           int32_t stalled_block, uint32_t limit_cycles) {
    if (stalled_block < 0 || limit_cycles == 0) {
        g_last_error = "stalled_block must be >= 0 and limit_cycles > 0";
        return DG_ERR_INVALID_ARG;
    }
    return selfcond_impl(logits, logits_dtype, ld, B, C, V, inv_tau, lse, E, embed_dtype, d, z, workspace,
                         workspace_bytes, stream, stalled_block, static_cast<long long>(limit_cycles));
}


int dg_tau_linear(const double* t, int32_t B, double tau_max, double tau_min, float* inv_tau) {
    g_last_error.clear();
    if (!t || !inv_tau) return fail(DG_ERR_INVALID_ARG, "t and inv_tau (host arrays) are required");
    if (B < 1) return fail(DG_ERR_INVALID_ARG, "B = %d must be >= 1", B);
    if (!(tau_min > 0.0) || !(tau_max > 0.0) || !std::isfinite(tau_min) || !std::isfinite(tau_max))
        return fail(DG_ERR_INVALID_ARG, "tau_max = %g and tau_min = %g must be finite and > 0", tau_max, tau_min);
    for (int32_t b = 0; b < B; ++b) {
        double x = t[b];
        if (std::isnan(x)) return fail(DG_ERR_INVALID_ARG, "t[%d] is NaN", b);
        x = x < 0.0 ? 0.0 : (x > 1.0 ? 1.0 : x);
        inv_tau[b] = static_cast<float>(1.0 / (tau_min + (tau_max - tau_min) * x));
    }
    return DG_OK;
}

int dg_entropy_accept(const float* entropy, const int32_t* x0_hat, int32_t B, int32_t C, int32_t V, double eps,
                      uint64_t seed, uint32_t step, int32_t* x_next, uint8_t* accepted, int32_t* n_accepted,
                      dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if (!entropy || !x0_hat || !x_next) return fail(DG_ERR_INVALID_ARG, "entropy, x0_hat and x_next are required");
    if ((rc = check_canvases(B, C)) != DG_OK) return rc;
    if (C > DG_MAX_CANVAS_ROWS) return fail(DG_ERR_UNSUPPORTED, "C = %d exceeds %d", C, DG_MAX_CANVAS_ROWS);
    if (V < 1) return fail(DG_ERR_INVALID_ARG, "V = %d must be >= 1", V);
    if (std::isnan(eps)) return fail(DG_ERR_INVALID_ARG, "eps is NaN");
    if ((rc = check_device()) != DG_OK) return rc;
    DecideParams p;
    std::memset(&p, 0, sizeof(p));
    p.entropy = entropy;
    p.x0_hat = x0_hat;
    p.C = C;
    p.V = V;
    p.accept_limit = entropy_threshold(eps);
    p.key0 = static_cast<uint32_t>(seed);
    p.key1 = static_cast<uint32_t>(seed >> 32);
    p.step = step;
    p.x_next = x_next;
    p.accepted = accepted;
    p.n_accepted = n_accepted;
    const cudaError_t e = launch_canvas_decide(p, B, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "acceptance launch");
    return DG_OK;
}

int dg_adaptive_stop(const float* entropy, const int32_t* argmax, const int32_t* argmax_prev, int32_t B, int32_t C,
                     double theta, uint8_t* stop, float* mean_entropy, dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if (!entropy || !argmax) return fail(DG_ERR_INVALID_ARG, "entropy and argmax are required");
    if (!stop && !mean_entropy) return fail(DG_ERR_INVALID_ARG, "no output requested");
    if ((rc = check_canvases(B, C)) != DG_OK) return rc;
    if (C > DG_MAX_CANVAS_ROWS) return fail(DG_ERR_UNSUPPORTED, "C = %d exceeds %d", C, DG_MAX_CANVAS_ROWS);
    if (std::isnan(theta)) return fail(DG_ERR_INVALID_ARG, "theta is NaN");
    if ((rc = check_device()) != DG_OK) return rc;
    DecideParams p;
    std::memset(&p, 0, sizeof(p));
    p.entropy = entropy;
    p.argmax = argmax;
    p.argmax_prev = argmax_prev;
    p.C = C;
    p.stop_limit = entropy_threshold(theta * static_cast<double>(C));
    p.stop = stop;
    p.mean_entropy = mean_entropy;
    const cudaError_t e = launch_canvas_decide(p, B, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "stopping launch");
    return DG_OK;
}

int dg_sampler_step_eb(const void* logits, int logits_dtype, int64_t ld, int32_t B, int32_t C, int32_t V,
                       const float* inv_tau, uint64_t seed, uint32_t step, int x0_mode, double eps, double theta,
                       const int32_t* argmax_prev, int32_t* x_next, int32_t* x0_hat, int32_t* argmax,
                       float* max_prob, float* lse, float* entropy, uint8_t* accepted, uint8_t* stop,
                       float* mean_entropy, void* workspace, size_t workspace_bytes, dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if ((rc = check_logits(logits, logits_dtype, ld, V)) != DG_OK) return rc;
    if ((rc = check_canvases(B, C)) != DG_OK) return rc;
    if (C > DG_MAX_CANVAS_ROWS) return fail(DG_ERR_UNSUPPORTED, "C = %d exceeds %d", C, DG_MAX_CANVAS_ROWS);
    if (!x_next || !x0_hat || !entropy) return fail(DG_ERR_INVALID_ARG, "x_next, x0_hat and entropy are required");
    if ((stop || mean_entropy) && !argmax) return fail(DG_ERR_INVALID_ARG, "stopping needs the argmax output");
    if (x0_mode != DG_X0_SAMPLE && x0_mode != DG_X0_GREEDY)
        return fail(DG_ERR_INVALID_ARG, "x0_mode %d is not SAMPLE or GREEDY", x0_mode);
    if (std::isnan(eps) || std::isnan(theta)) return fail(DG_ERR_INVALID_ARG, "eps and theta may not be NaN");
    const int32_t R = B * C;
    const size_t need = pass_ws_bytes(R, V, 0);
    if (!workspace || workspace_bytes < need)
        return fail(DG_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
    if (!aligned16(workspace)) return fail(DG_ERR_ALIGNMENT, "workspace is not 16-byte aligned");
    static thread_local PassParams p;
    std::memset(&p, 0, sizeof(p));
    if ((rc = check_inv_tau(inv_tau, B, p.inv_tau)) != DG_OK) return rc;
    if ((rc = check_device()) != DG_OK) return rc;
    const PassWs w = carve_pass_ws(workspace, R, 0);
    p.logits = logits;
    p.ld = ld;
    p.R = R;
    p.C = C;
    p.V = V;
    p.n_chunks = n_chunks_of(V);
    p.groups_per_cta = groups_per_cta_of(n_groups_of(V));
    p.segs = (n_groups_of(V) + p.groups_per_cta - 1) / p.groups_per_cta;
    p.rec = w.rec;
    p.epoch = w.epoch;
    p.key0 = static_cast<uint32_t>(seed);
    p.key1 = static_cast<uint32_t>(seed >> 32);
    p.step = step;
    p.mode = x0_mode;
    p.x0_hat = x0_hat;  // x_next stays null: the per-canvas rule below decides it
    p.argmax = argmax;
    p.max_prob = max_prob;
    p.lse = lse;
    p.entropy = entropy;
    const cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = launch_logits_pass(p, kPassSampler, logits_dtype == DG_BF16, st);
    if (e != cudaSuccess) return cuda_fail(e, "logits pass launch");
    DecideParams d;
    std::memset(&d, 0, sizeof(d));
    d.entropy = entropy;
    d.x0_hat = x0_hat;
    d.argmax = argmax;
    d.argmax_prev = argmax_prev;
    d.C = C;
    d.V = V;
    d.accept_limit = entropy_threshold(eps);
    d.stop_limit = entropy_threshold(theta * static_cast<double>(C));
    d.key0 = p.key0;
    d.key1 = p.key1;
    d.step = step;
    d.x_next = x_next;
    d.accepted = accepted;
    d.stop = stop;
    d.mean_entropy = mean_entropy;
    e = launch_canvas_decide(d, B, st);
    if (e != cudaSuccess) return cuda_fail(e, "per-canvas decision launch");
    return DG_OK;
}

int dg_canvas_ce_backward(void* logits, int64_t ld, const float* lse_rows, const int32_t* x0,
                          const int32_t* canvas_idx, int32_t n_seq, int32_t P, int32_t K, int32_t C, int32_t V,
                          const float* g_seq, dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if ((rc = check_logits(logits, DG_BF16, ld, V)) != DG_OK) return rc;
    if (!lse_rows || !x0 || !canvas_idx) return fail(DG_ERR_INVALID_ARG, "lse_rows, x0 and canvas_idx are required");
    if (n_seq < 1 || n_seq > DG_MAX_CANVASES)
        return fail(DG_ERR_INVALID_ARG, "n_seq = %d must be in [1, %d]", n_seq, DG_MAX_CANVASES);
    if (P < 0 || K < 1 || C < 1) return fail(DG_ERR_INVALID_ARG, "need P >= 0, K >= 1, C >= 1");
    if (V % 8 != 0) return fail(DG_ERR_ALIGNMENT, "V = %d must be a multiple of 8 (16-byte bf16 vectors)", V);
    const long long L = static_cast<long long>(P) + static_cast<long long>(K) * C;
    if (L > 0x7fffffffLL || static_cast<long long>(n_seq) * C > 0x7fffffffLL)
        return fail(DG_ERR_INVALID_ARG, "sizes overflow int32");
    if ((rc = check_device()) != DG_OK) return rc;
    CeBackwardParams p;
    std::memset(&p, 0, sizeof(p));
    p.logits = logits;
    p.ld = ld;
    p.lse = lse_rows;
    p.x0 = x0;
    p.canvas_idx = canvas_idx;
    p.g_seq = g_seq;
    p.R = n_seq * C;
    p.C = C;
    p.V = V;
    p.P = P;
    p.K = K;
    p.seq_len = L;
    const cudaError_t e = launch_ce_backward(p, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "CE backward launch");
    return DG_OK;
}

int dg_selfcond_drop(void* z, int32_t n_seq, int32_t C, int32_t d, uint64_t seed, uint32_t step, uint8_t* keep,
                     dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if (!z) return fail(DG_ERR_INVALID_ARG, "z is NULL");
    if (n_seq < 1 || C < 1 || d < 1) return fail(DG_ERR_INVALID_ARG, "need n_seq, C, d >= 1");
    if (!aligned16(z)) return fail(DG_ERR_ALIGNMENT, "z is not 16-byte aligned");
    const long long per_seq = static_cast<long long>(C) * d;
    if (per_seq % 8 != 0) return fail(DG_ERR_ALIGNMENT, "C * d = %lld must be a multiple of 8", per_seq);
    if ((rc = check_device()) != DG_OK) return rc;
    const cudaError_t e = launch_selfcond_drop(static_cast<uint16_t*>(z), n_seq, per_seq, static_cast<uint32_t>(seed),
                                               static_cast<uint32_t>(seed >> 32), step, keep,
                                               reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "self-conditioning drop launch");
    return DG_OK;
}


size_t dg_ffw_workspace_size(int32_t rows, int32_t d, int32_t d_ff) {
    if (rows < 1 || d < 64 || d_ff < 64) return 0;
    const size_t a = selfcond_partial_bytes(rows, d, d_ff, true, true);  // layer 1: K = d, N = d_ff
    const size_t b = selfcond_partial_bytes(rows, d_ff, d, true, true);  // layer 2: K = d_ff, N = d
    return a > b ? a : b;
}

int dg_ffw(const void* z_in, int32_t rows, int32_t d, int32_t d_ff, const void* W1, const void* W2, void* hidden,
           void* z_out, void* workspace, size_t workspace_bytes, dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if (!z_in || !W1 || !W2 || !hidden || !z_out)
        return fail(DG_ERR_INVALID_ARG, "z_in, W1, W2, hidden and z_out are required");
    if (rows < 1) return fail(DG_ERR_INVALID_ARG, "rows = %d must be >= 1", rows);
    if (d < 64 || d > 16384 || d % 64 != 0 || d_ff < 64 || d_ff > 16384 || d_ff % 64 != 0)
        return fail(DG_ERR_INVALID_ARG, "d = %d and d_ff = %d must be multiples of 64 in [64, 16384]", d, d_ff);
    if (!aligned16(z_in) || !aligned16(W1) || !aligned16(W2) || !aligned16(hidden) || !aligned16(z_out))
        return fail(DG_ERR_ALIGNMENT, "all operands must be 16-byte aligned");
    if (z_in == z_out || hidden == z_in || hidden == z_out)
        return fail(DG_ERR_INVALID_ARG, "z_in, hidden and z_out may not alias");
    const size_t need = dg_ffw_workspace_size(rows, d, d_ff);
    if (need && (!workspace || workspace_bytes < need))
        return fail(DG_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
    if (need && (reinterpret_cast<uintptr_t>(workspace) & 255u))
        return fail(DG_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
    if ((rc = check_device()) != DG_OK) return rc;
    const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    static thread_local SelfcondParams sp;
    for (int layer = 0; layer < 2; ++layer) {
        std::memset(&sp, 0, sizeof(sp));
        sp.logits = layer == 0 ? z_in : hidden;
        sp.ld = layer == 0 ? d : d_ff;
        sp.logits_bf16 = 1;
        sp.E = static_cast<const uint16_t*>(layer == 0 ? W1 : W2);
        sp.z = static_cast<uint16_t*>(layer == 0 ? hidden : z_out);
        sp.R = rows;
        sp.C = rows;
        sp.V = layer == 0 ? d : d_ff;
        sp.d = layer == 0 ? d_ff : d;
        sp.partial = static_cast<float*>(workspace);
        sp.fault_block = -1;
        sp.plain_a = 1;
        sp.act = layer == 0 ? 1 : 0;
        sp.inv_tau[0] = 1.0f;
        // the second layer may be placed while the first drains: its weight copies start at once,
        // its hidden-layer copies wait for the preceding grid
        sp.dependent = layer == 1 ? 1 : 0;
        const cudaError_t e = launch_selfcond(sp, s);
        if (e != cudaSuccess) return cuda_fail(e, layer == 0 ? "FFW layer 1 launch" : "FFW layer 2 launch");
    }
    return DG_OK;
}


int dg_sampler_selfcond_step(const void* logits, int logits_dtype, int64_t ld, const int32_t* x_t, int32_t B,
                             int32_t C, int32_t V, int schedule, const double* t, const double* dt,
                             const float* inv_tau, uint64_t seed, uint32_t step, int x0_mode, int32_t* x_next,
                             int32_t* x0_hat, int32_t* argmax, float* max_prob, float* lse, float* entropy,
                             uint8_t* branch, void* workspace, size_t workspace_bytes, const void* E,
                             int embed_dtype, int32_t d, void* z, void* z_workspace, size_t z_workspace_bytes,
                             dg_stream_t stream) {
    if (!lse) {
        g_last_error = "lse is required (the contraction reads it)";
        return DG_ERR_INVALID_ARG;
    }
    // every argument of the contraction is checked before the logits pass is launched
    int rc = selfcond_impl(logits, logits_dtype, ld, B, C, V, inv_tau, lse, E, embed_dtype, d, z, z_workspace,
                           z_workspace_bytes, stream, -1, 0, false, true);
    if (rc != DG_OK) return rc;
    rc = dg_sampler_step(logits, logits_dtype, ld, x_t, B, C, V, schedule, t, dt, inv_tau, seed, step, x0_mode,
                         x_next, x0_hat, argmax, max_prob, lse, entropy, branch, workspace, workspace_bytes, stream);
    if (rc != DG_OK) return rc;
    return selfcond_impl(logits, logits_dtype, ld, B, C, V, inv_tau, lse, E, embed_dtype, d, z, z_workspace,
                         z_workspace_bytes, stream, -1, 0, true, false);
}


int dg_test_merge_stall(const void* logits, int logits_dtype, int64_t ld, int32_t rows, int32_t V, float* lse,
                        void* workspace, size_t workspace_bytes, uint32_t limit_cycles, dg_stream_t stream) {
    g_last_error.clear();
    int rc;
    if ((rc = check_logits(logits, logits_dtype, ld, V)) != DG_OK) return rc;
    if (rows < 1 || !lse) return fail(DG_ERR_INVALID_ARG, "rows >= 1 and lse are required");
    if (limit_cycles == 0) return fail(DG_ERR_INVALID_ARG, "limit_cycles must be > 0");
    const size_t need = pass_ws_bytes(rows, V, 0);
    if (!workspace || workspace_bytes < need)
        return fail(DG_ERR_WORKSPACE, "workspace of %zu bytes is smaller than the %zu required", workspace_bytes, need);
    if ((rc = check_device()) != DG_OK) return rc;
    static thread_local PassParams p;
    std::memset(&p, 0, sizeof(p));
    const PassWs w = carve_pass_ws(workspace, rows, 0);
    p.logits = logits;
    p.ld = ld;
    p.R = rows;
    p.C = rows;
    p.V = V;
    p.n_chunks = n_chunks_of(V);
    p.groups_per_cta = groups_per_cta_of(n_groups_of(V));
    p.segs = (n_groups_of(V) + p.groups_per_cta - 1) / p.groups_per_cta;
    p.rec = w.rec;
    p.epoch = w.epoch;
    p.lse = lse;
    p.inv_tau[0] = 1.0f;
    p.merge_wait_limit = static_cast<long long>(limit_cycles);
    const cudaError_t e = launch_merge_only(p, logits_dtype == DG_BF16, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "merge stall test launch");
    return DG_OK;
}

}  // extern "C"
