// gdr_lib.cu -- the C ABI of libgdr.so (declared in include/gdr.h): argument
// validation, workspace sizing, kernel selection and the device status word.
// Every kernel header is included here so the library is one translation
// unit (the device status word is then a single symbol).
#include <stdarg.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <mutex>
#include <string>

#include "common.cuh"
#include "step_kernel.cuh"
#include "fwd_simt.cuh"
#include "bwd_simt.cuh"
#include "block.cuh"
#include "seg_split.cuh"
#include "gdr2_simt.cuh"
#include "fwd_tc.cuh"
#include "fwd_tc2.cuh"
#include "bwd_tc.cuh"
#include "fwd2_tc.cuh"
#include "fwd2_tc2.cuh"
#include "bwd2_simt.cuh"

namespace gdr {
std::atomic<uint64_t> g_launches{0};
}  // namespace gdr

using namespace gdr;

namespace {

thread_local std::string t_last_error;

gdr_status fail(gdr_status s, const char *fmt, ...) __attribute__((format(printf, 2, 3)));
gdr_status fail(gdr_status s, const char *fmt, ...) {
    char buf[512];
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(buf, sizeof(buf), fmt, ap);
    va_end(ap);
    t_last_error = buf;
    return s;
}

gdr_status cuda_fail(cudaError_t e, const char *where) {
    return fail(GDR_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

#define GDR_REQUIRE_PTR(p)                                                                   \
    do {                                                                                     \
        if ((p) == nullptr) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: %s is NULL", fn, #p); \
        if (!aligned16(p))                                                                   \
            return fail(GDR_ERR_INVALID_ARGUMENT, "%s: %s is not 16-byte aligned", fn, #p);  \
    } while (0)
#define GDR_OPTIONAL_PTR(p)                                                                 \
    do {                                                                                    \
        if ((p) != nullptr && !aligned16(p))                                                \
            return fail(GDR_ERR_INVALID_ARGUMENT, "%s: %s is not 16-byte aligned", fn, #p); \
    } while (0)

gdr_status check_dims(const char *fn, int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    if (B < 1 || T < 1 || H < 1 || dk < 1 || dv < 1)
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: sizes must be positive (B=%d T=%d H=%d dk=%d dv=%d)",
                    fn, B, T, H, dk, dv);
    if (dt != GDR_F32 && dt != GDR_BF16)
        return fail(GDR_ERR_UNSUPPORTED, "%s: unknown dtype %d", fn, (int)dt);
    if ((dk != 64 && dk != 128) || (dv != 64 && dv != 128))
        return fail(GDR_ERR_UNSUPPORTED, "%s: dk=%d dv=%d (supported: 64 or 128 each)", fn, dk, dv);
    const long long elems = (long long)B * T * H * (dk > dv ? dk : dv);
    if (elems >= (1LL << 31))
        return fail(GDR_ERR_UNSUPPORTED, "%s: B*T*H*max(dk,dv) = %lld exceeds 2^31-1", fn, elems);
    if ((long long)B * H * (dv / 64) >= (1LL << 31))
        return fail(GDR_ERR_UNSUPPORTED, "%s: too many (batch, head) units", fn);
    return GDR_OK;
}


// bf16 with dk = dv = 128 runs the backward on the tensor cores (recompute,
// dS pass, chunk-parallel gradients); GDR_BWD_KERNEL=simt selects the
// CUDA-core backward (used to cross-check them).  The workspace size follows
// the same choice.
bool bwd_uses_tc(int dk, int dv, gdr_dtype dt) {
    const char *sel = getenv("GDR_BWD_KERNEL");
    return dt == GDR_BF16 && dk == 128 && dv == 128 && !(sel != nullptr && strcmp(sel, "simt") == 0);
}
size_t bwd_scratch_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    return bwd_uses_tc(dk, dv, dt) ? 2 * bwd_tc_state_bytes(B, T, H) : bwd_workspace_bytes(B, T, H, dk, dv);
}

// The backward's kernels for one call (shared by gdr_bwd and gdr_bwd_noalloc).
cudaError_t run_bwd(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                    const void *v, const float *log_alpha, const float *beta, const float *S0, const void *dO,
                    const float *dS_T, void *dq, void *dk_out, void *dv_out, float *dlog_alpha, float *dbeta,
                    float *dS0, void *workspace, cudaStream_t s) {
    if (bwd_uses_tc(dk, dv, dt))
        return launch_bwd_tc(B, T, H, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk_out, dv_out, dlog_alpha,
                             dbeta, dS0, workspace, s);
#define GDR_BWD_ARGS B, T, H, dv, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk_out, dv_out, \
                     dlog_alpha, dbeta, dS0, workspace, s
    if (dt == GDR_F32)
        return dk == 128 ? launch_bwd_simt<float, 128>(GDR_BWD_ARGS) : launch_bwd_simt<float, 64>(GDR_BWD_ARGS);
    return dk == 128 ? launch_bwd_simt<__nv_bfloat16, 128>(GDR_BWD_ARGS)
                     : launch_bwd_simt<__nv_bfloat16, 64>(GDR_BWD_ARGS);
#undef GDR_BWD_ARGS
}
}  // namespace

extern "C" {

int gdr_version(void) { return (0 << 16) | 1; }

uint64_t gdr_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

const char *gdr_last_error_string(void) { return t_last_error.c_str(); }

gdr_status gdr_check_status(gdr_stream_t stream) {
    cudaError_t e = cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, "gdr_check_status: synchronize");
    int host = 0, zero = 0;
    e = cudaMemcpyFromSymbol(&host, g_status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "gdr_check_status: read status");
    if (host != 0) {
        e = cudaMemcpyToSymbol(g_status, &zero, sizeof(int));
        if (e != cudaSuccess) return cuda_fail(e, "gdr_check_status: clear status");
        return fail((gdr_status)host, "device status %d: %s", host,
                    host == GDR_ERR_TIMEOUT ? "a bounded on-chip wait gave up"
                                            : "a kernel reported an input it does not handle");
    }
    return GDR_OK;
}

// One thread waits, with a short bound, on a barrier that never completes.
__global__ void gdr_timeout_probe_kernel(uint64_t limit_ns) {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        sm100::mbar_init(&bar, 1);
        sm100::fence_mbar_init();
        if (!sm100::mbar_wait(&bar, 0, limit_ns)) record_status(GDR_ERR_TIMEOUT);
    }
}

gdr_status gdr_debug_wait_timeout(int timeout_ms, gdr_stream_t stream) {
    const char *fn = "gdr_debug_wait_timeout";
    if (timeout_ms < 1 || timeout_ms > 10000)
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: timeout_ms=%d (1..10000)", fn, timeout_ms);
    gdr_timeout_probe_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        (uint64_t)timeout_ms * 1000000ull);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    cudaError_t e = cudaGetLastError();
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

// The two passes of gdr_seg_fwd are independent; the second runs on an
// auxiliary stream of the device (created on first use, with a fork and a
// join event), so the two small grids share the GPU.  The enqueue sequence is
// serialised by a mutex so the events can be reused.
struct SegAux {
    cudaStream_t stream = nullptr;
    cudaEvent_t fork = nullptr, join = nullptr;
};
std::mutex g_seg_mu;
SegAux g_seg_aux[64];

// The device's auxiliary stream and events (created on first use); call with
// g_seg_mu held.
cudaError_t seg_aux(SegAux **out) {
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    SegAux &aux = g_seg_aux[dev];
    if (aux.stream == nullptr) {
        e = cudaStreamCreateWithFlags(&aux.stream, cudaStreamNonBlocking);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&aux.fork, cudaEventDisableTiming);
        if (e == cudaSuccess) e = cudaEventCreateWithFlags(&aux.join, cudaEventDisableTiming);
        if (e != cudaSuccess) return e;
    }
    *out = &aux;
    return cudaSuccess;
}

// One sequence on one GPU as R segments (gdr_fwd for bf16, dk = dv = 128):
// a B-batch sequence viewed as [B*R, T/R, H, d] runs both passes of the
// sequence split concurrently -- pass 1 from S_in = 0 into o and N, pass 2
// with v = 0 from S_in = I into q~ and M -- then the scan of the segment
// maps and the tensor-core correction o += S_in q~.  Used when the two
// passes still fit the SMs in one wave (4 B H R <= SMs: each (b, h) of the
// forward is a cluster of two CTAs) and every segment has at least
// kSplitMinTokens tokens.
constexpr int kSplitMinTokens = 2048;

int fwd_split_r(int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    if (dt != GDR_BF16 || dk != 128 || dv != 128) return 1;
    const char *sel = getenv("GDR_FWD_SPLIT");
    if (sel != nullptr && strcmp(sel, "off") == 0) return 1;
    const char *ksel = getenv("GDR_FWD_KERNEL");
    if (ksel != nullptr) return 1;  // a forced kernel runs unsplit
    int dev = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 1;
    for (int R = sms / (4 * B * H); R >= 2; --R)
        if (T % R == 0 && T / R >= kSplitMinTokens) return R;
    return 1;
}

struct SplitWs {
    size_t zero_v, eye, qt, N, M, S_in, total;
};
SplitWs split_ws(int B, int T, int H, int R) {
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    SplitWs w;
    const size_t tok = (size_t)B * T * H * 128 * 2, st = (size_t)B * R * H * 128 * 128 * 4;
    w.zero_v = 0;
    w.eye = al(tok);
    w.qt = w.eye + al(st);
    w.N = w.qt + al(tok);
    w.M = w.N + al(st);
    w.S_in = w.M + al(st);
    w.total = w.S_in + al(st);
    return w;
}

size_t gdr_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    if (B < 1 || T < 1 || H < 1) return 0;
    const int R = fwd_split_r(B, T, H, dk, dv, dt);
    return R > 1 ? split_ws(B, T, H, R).total : 0;
}

// The split forward (see fwd_split_r); o, S_T as for gdr_fwd.
gdr_status run_fwd_split(int B, int T, int H, int R, const void *q, const void *k, const void *v,
                         const float *la, const float *beta, const float *S0, void *o, float *S_T, void *workspace,
                         cudaStream_t s) {
    const char *fn = "gdr_fwd";
    const SplitWs w = split_ws(B, T, H, R);
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    void *zero_v = ws + w.zero_v, *qt = ws + w.qt;
    float *eye = reinterpret_cast<float *>(ws + w.eye), *N = reinterpret_cast<float *>(ws + w.N);
    float *M = reinterpret_cast<float *>(ws + w.M), *S_in = reinterpret_cast<float *>(ws + w.S_in);
    const int Bs = B * R, Ts = T / R;
    std::lock_guard<std::mutex> lock(g_seg_mu);
    SegAux *aux = nullptr;
    cudaError_t e = seg_aux(&aux);
    if (e == cudaSuccess) e = cudaEventRecord(aux->fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(aux->stream, aux->fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    // pass 1 (caller's stream) and pass 2 (auxiliary stream)
    cudaError_t e1 = launch_fwd_tc2(Bs, Ts, H, q, k, v, la, beta, nullptr, o, N, s);
    // With S0 = 0 and one batch, segment 0 needs neither q~ (its S_in is 0)
    // nor M (segment 1 starts from N_0): pass 2 covers segments 1 .. R-1.
    const int m0 = (S0 == nullptr && B == 1) ? 1 : 0;
    const size_t tok_seg = (size_t)Ts * H * 128;  // elements of one segment
    cudaError_t e2 = cudaMemsetAsync(zero_v, 0, (size_t)(Bs - m0) * tok_seg * 2, aux->stream);
    if (e2 == cudaSuccess) e2 = launch_seg_identity(eye, (Bs - m0) * H, 128, aux->stream);
    if (e2 == cudaSuccess)
        e2 = launch_fwd_tc2(Bs - m0, Ts, H, static_cast<const __nv_bfloat16 *>(q) + m0 * tok_seg,
                            static_cast<const __nv_bfloat16 *>(k) + m0 * tok_seg, zero_v, la + m0 * (size_t)Ts * H,
                            beta + m0 * (size_t)Ts * H, eye, static_cast<__nv_bfloat16 *>(qt) + m0 * tok_seg,
                            M + m0 * (size_t)H * 128 * 128, aux->stream);
    cudaError_t ej = cudaEventRecord(aux->join, aux->stream);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, aux->join, 0);
    if (e1 != cudaSuccess) return cuda_fail(e1, fn);
    if (e2 != cudaSuccess) return cuda_fail(e2, fn);
    if (ej != cudaSuccess) return cuda_fail(ej, fn);
    // scan of the segment maps, then o += S_in q~
    e = launch_seg_scan(B, R, H, 128, 128, M, N, S0, S_in, S_T, s);
    // with S0 = 0 the first segment of every batch has S_in = 0: skip it
    if (e == cudaSuccess) e = launch_seg_fixup_tc(B, Ts, H, qt, S_in, o, s, R, S0 == nullptr ? 1 : 0);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}


gdr_status gdr_fwd(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                   const void *v, const float *log_alpha, const float *beta, const float *S0,
                   void *o, float *S_T, void *workspace, size_t workspace_bytes,
                   gdr_stream_t stream) {
    const char *fn = "gdr_fwd";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(beta);
    GDR_REQUIRE_PTR(o);
    GDR_OPTIONAL_PTR(S0);
    GDR_OPTIONAL_PTR(S_T);
    GDR_OPTIONAL_PTR(workspace);
    // The workspace is optional: with at least gdr_fwd_workspace_bytes a long
    // sequence over few heads runs as parallel segments, otherwise unsplit.
    const size_t need = gdr_fwd_workspace_bytes(B, T, H, dk, dv, dt);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    // a long sequence over few (b, h): segments of the sequence in parallel
    // (only with the workspace gdr_fwd_workspace_bytes asks for)
    if (need > 0 && workspace != nullptr && workspace_bytes >= need) {
        const int R = fwd_split_r(B, T, H, dk, dv, dt);
        if (R > 1) return run_fwd_split(B, T, H, R, q, k, v, log_alpha, beta, S0, o, S_T, workspace, s);
    }
    // bf16 with dk = dv = 128 runs on the tensor cores (the two-SM cluster
    // kernel); GDR_FWD_KERNEL=tc1 selects the single-CTA tensor-core kernel and
    // GDR_FWD_KERNEL=simt the CUDA-core kernel (used to cross-check them).
    const char *sel = getenv("GDR_FWD_KERNEL");
    const bool force_simt = sel != nullptr && strcmp(sel, "simt") == 0;
    const bool force_tc1 = sel != nullptr && strcmp(sel, "tc1") == 0;
    if (dt == GDR_BF16 && dk == 128 && dv == 128 && !force_simt) {
        e = force_tc1 ? launch_fwd_tc(B, T, H, q, k, v, log_alpha, beta, S0, o, S_T, s)
                      : launch_fwd_tc2(B, T, H, q, k, v, log_alpha, beta, S0, o, S_T, s);
        if (e != cudaSuccess) return cuda_fail(e, fn);
        return GDR_OK;
    }
    if (dt == GDR_F32)
        e = dk == 128 ? launch_fwd_simt<float, 128>(B, T, H, dv, q, k, v, log_alpha, beta, S0, o, S_T, s)
                      : launch_fwd_simt<float, 64>(B, T, H, dv, q, k, v, log_alpha, beta, S0, o, S_T, s);
    else
        e = dk == 128
                ? launch_fwd_simt<__nv_bfloat16, 128>(B, T, H, dv, q, k, v, log_alpha, beta, S0, o, S_T, s)
                : launch_fwd_simt<__nv_bfloat16, 64>(B, T, H, dv, q, k, v, log_alpha, beta, S0, o, S_T, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

gdr_status gdr_step(int B, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                    const void *v, const float *log_alpha, const float *beta, float *S, void *o,
                    gdr_stream_t stream) {
    const char *fn = "gdr_step";
    gdr_status st = check_dims(fn, B, 1, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(beta);
    GDR_REQUIRE_PTR(S);
    GDR_REQUIRE_PTR(o);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == GDR_F32)
        e = dk == 128 ? launch_step<float, 128>(B, H, dv, q, k, v, log_alpha, beta, S, o, s)
                      : launch_step<float, 64>(B, H, dv, q, k, v, log_alpha, beta, S, o, s);
    else
        e = dk == 128 ? launch_step<__nv_bfloat16, 128>(B, H, dv, q, k, v, log_alpha, beta, S, o, s)
                      : launch_step<__nv_bfloat16, 64>(B, H, dv, q, k, v, log_alpha, beta, S, o, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

gdr_status gdr2_step(int B, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                     const void *v, const float *log_alpha, const float *b, const float *w, float *S, void *o,
                     gdr_stream_t stream) {
    const char *fn = "gdr2_step";
    gdr_status st = check_dims(fn, B, 1, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(b);
    GDR_REQUIRE_PTR(w);
    GDR_REQUIRE_PTR(S);
    GDR_REQUIRE_PTR(o);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    if (dt == GDR_F32)
        e = dk == 128 ? launch_step2<float, 128>(B, H, dv, q, k, v, log_alpha, b, w, S, o, s)
                      : launch_step2<float, 64>(B, H, dv, q, k, v, log_alpha, b, w, S, o, s);
    else
        e = dk == 128 ? launch_step2<__nv_bfloat16, 128>(B, H, dv, q, k, v, log_alpha, b, w, S, o, s)
                      : launch_step2<__nv_bfloat16, 64>(B, H, dv, q, k, v, log_alpha, b, w, S, o, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

size_t gdr_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    if (B < 1 || T < 1 || H < 1 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    return bwd_scratch_bytes(B, T, H, dk, dv, dt);
}

gdr_status gdr_bwd(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                   const void *v, const float *log_alpha, const float *beta, const float *S0,
                   const void *dO, const float *dS_T, void *dq, void *dk_out, void *dv_out,
                   float *dlog_alpha, float *dbeta, float *dS0, void *workspace,
                   size_t workspace_bytes, gdr_stream_t stream) {
    const char *fn = "gdr_bwd";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(beta);
    GDR_REQUIRE_PTR(dO);
    GDR_REQUIRE_PTR(dq);
    GDR_REQUIRE_PTR(dk_out);
    GDR_REQUIRE_PTR(dv_out);
    GDR_REQUIRE_PTR(dlog_alpha);
    GDR_REQUIRE_PTR(dbeta);
    GDR_OPTIONAL_PTR(S0);
    GDR_OPTIONAL_PTR(dS_T);
    GDR_OPTIONAL_PTR(dS0);
    const size_t need = gdr_bwd_workspace_bytes(B, T, H, dk, dv, dt);
    if (workspace == nullptr || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned16(workspace))
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: workspace is not 16-byte aligned", fn);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    e = run_bwd(B, T, H, dk, dv, dt, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk_out, dv_out, dlog_alpha,
                dbeta, dS0, workspace, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

size_t gdr2_fwd_workspace_bytes(int, int, int, int, int, gdr_dtype) { return 0; }

gdr_status gdr2_fwd(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                    const void *v, const float *log_alpha, const float *b, const float *w,
                    const float *S0, void *o, float *S_T, void *workspace, size_t workspace_bytes,
                    gdr_stream_t stream) {
    const char *fn = "gdr2_fwd";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(b);
    GDR_REQUIRE_PTR(w);
    GDR_REQUIRE_PTR(o);
    GDR_OPTIONAL_PTR(S0);
    GDR_OPTIONAL_PTR(S_T);
    GDR_OPTIONAL_PTR(workspace);
    (void)workspace_bytes;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
    // bf16 with dk = dv = 128 runs on the tensor cores (the two-SM cluster
    // kernel); GDR2_FWD_KERNEL=tc1 selects the single-CTA tensor-core kernel
    // and GDR2_FWD_KERNEL=simt the CUDA-core kernel (used to cross-check them).
    const char *sel = getenv("GDR2_FWD_KERNEL");
    if (dt == GDR_BF16 && dk == 128 && dv == 128 && !(sel != nullptr && strcmp(sel, "simt") == 0)) {
        const bool tc1 = sel != nullptr && strcmp(sel, "tc1") == 0;
        e = tc1 ? launch_fwd2_tc(B, T, H, q, k, v, log_alpha, b, w, S0, o, S_T, s)
                : launch_fwd2_tc2(B, T, H, q, k, v, log_alpha, b, w, S0, o, S_T, s);
        if (e != cudaSuccess) return cuda_fail(e, fn);
        return GDR_OK;
    }
#define GDR2_ARGS B, T, H, dv, q, k, v, log_alpha, b, w, S0, o, S_T, s
    if (dt == GDR_F32)
        e = dk == 128 ? launch_gdr2_simt<float, 128>(GDR2_ARGS) : launch_gdr2_simt<float, 64>(GDR2_ARGS);
    else
        e = dk == 128 ? launch_gdr2_simt<__nv_bfloat16, 128>(GDR2_ARGS)
                      : launch_gdr2_simt<__nv_bfloat16, 64>(GDR2_ARGS);
#undef GDR2_ARGS
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

size_t gdr2_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    if (B < 1 || T < 1 || H < 1 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128)) return 0;
    return bwd2_workspace_bytes(B, T, H, dk, dv, dt == GDR_BF16);
}

gdr_status gdr2_bwd(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                    const void *v, const float *log_alpha, const float *b, const float *w, const float *S0,
                    const void *dO, const float *dS_T, void *dq, void *dk_out, void *dv_out, float *dlog_alpha,
                    float *db, float *dw, float *dS0, void *workspace, size_t workspace_bytes,
                    gdr_stream_t stream) {
    const char *fn = "gdr2_bwd";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(b);
    GDR_REQUIRE_PTR(w);
    GDR_REQUIRE_PTR(dO);
    GDR_REQUIRE_PTR(dq);
    GDR_REQUIRE_PTR(dk_out);
    GDR_REQUIRE_PTR(dv_out);
    GDR_REQUIRE_PTR(dlog_alpha);
    GDR_REQUIRE_PTR(db);
    GDR_REQUIRE_PTR(dw);
    GDR_OPTIONAL_PTR(S0);
    GDR_OPTIONAL_PTR(dS_T);
    GDR_OPTIONAL_PTR(dS0);
    const size_t need = bwd2_workspace_bytes(B, T, H, dk, dv, dt == GDR_BF16);
    if (workspace == nullptr || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need,
                    workspace ? workspace_bytes : (size_t)0);
    if (!aligned16(workspace))
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: workspace is not 16-byte aligned", fn);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e;
#define GDR2_BWD_ARGS B, T, H, dv, q, k, v, log_alpha, b, w, S0, dO, dS_T, dq, dk_out, dv_out, dlog_alpha, \
                      db, dw, dS0, workspace, s
    if (dt == GDR_F32)
        e = dk == 128 ? launch_bwd2_simt<float, 128>(GDR2_BWD_ARGS) : launch_bwd2_simt<float, 64>(GDR2_BWD_ARGS);
    else
        e = dk == 128 ? launch_bwd2_simt<__nv_bfloat16, 128>(GDR2_BWD_ARGS)
                      : launch_bwd2_simt<__nv_bfloat16, 64>(GDR2_BWD_ARGS);
#undef GDR2_BWD_ARGS
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

gdr_status gdr_block_prologue(int B, int T, int H, int dk, int dv, int K, gdr_dtype dt, const void *xq,
                              const void *xk, const void *xv, const float *wq, const float *wk,
                              const float *wv, const float *bq, const float *bk, const float *bv,
                              const void *conv_state_in, void *conv_state_out, float eps, void *q, void *k,
                              void *v, gdr_stream_t stream) {
    const char *fn = "gdr_block_prologue";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    if (K < 1 || K > kConvMax)
        return fail(GDR_ERR_UNSUPPORTED, "%s: conv width K=%d (supported: 1..%d)", fn, K, kConvMax);
    if (!(eps >= 0.f) || eps > 1e30f) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: eps=%g", fn, (double)eps);
    GDR_REQUIRE_PTR(xq);
    GDR_REQUIRE_PTR(xk);
    GDR_REQUIRE_PTR(xv);
    GDR_REQUIRE_PTR(wq);
    GDR_REQUIRE_PTR(wk);
    GDR_REQUIRE_PTR(wv);
    GDR_OPTIONAL_PTR(bq);
    GDR_OPTIONAL_PTR(bk);
    GDR_OPTIONAL_PTR(bv);
    GDR_OPTIONAL_PTR(conv_state_in);
    GDR_OPTIONAL_PTR(conv_state_out);
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    PrologueArgs a{};
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.K = K;
    a.x[0] = xq; a.x[1] = xk; a.x[2] = xv;
    a.w[0] = wq; a.w[1] = wk; a.w[2] = wv;
    a.bias[0] = bq; a.bias[1] = bk; a.bias[2] = bv;
    a.state_in = K > 1 ? conv_state_in : nullptr;
    a.state_out = K > 1 ? conv_state_out : nullptr;
    a.eps = eps;
    a.y[0] = q; a.y[1] = k; a.y[2] = v;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = dt == GDR_F32 ? launch_prologue<float>(a, s) : launch_prologue<__nv_bfloat16>(a, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

size_t gdr_block_prologue_bwd_workspace_bytes(int H, int dk, int dv, int K) {
    if (H < 1 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128) || K < 1 || K > kConvMax) return 0;
    return prologue_bwd_workspace(H, dk, dv, K);
}

gdr_status gdr_block_prologue_bwd(int B, int T, int H, int dk, int dv, int K, gdr_dtype dt, const void *xq,
                                  const void *xk, const void *xv, const float *wq, const float *wk,
                                  const float *wv, const float *bq, const float *bk, const float *bv,
                                  const void *conv_state_in, float eps, const void *dyq, const void *dyk,
                                  const void *dyv, const void *dconv_state_out, void *dxq, void *dxk, void *dxv,
                                  float *dwq, float *dwk, float *dwv, float *dbq, float *dbk, float *dbv,
                                  void *dconv_state_in, void *workspace, size_t workspace_bytes,
                                  gdr_stream_t stream) {
    const char *fn = "gdr_block_prologue_bwd";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    if (K < 1 || K > kConvMax)
        return fail(GDR_ERR_UNSUPPORTED, "%s: conv width K=%d (supported: 1..%d)", fn, K, kConvMax);
    if (!(eps >= 0.f) || eps > 1e30f) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: eps=%g", fn, (double)eps);
    GDR_REQUIRE_PTR(xq);
    GDR_REQUIRE_PTR(xk);
    GDR_REQUIRE_PTR(xv);
    GDR_REQUIRE_PTR(wq);
    GDR_REQUIRE_PTR(wk);
    GDR_REQUIRE_PTR(wv);
    GDR_OPTIONAL_PTR(bq);
    GDR_OPTIONAL_PTR(bk);
    GDR_OPTIONAL_PTR(bv);
    GDR_OPTIONAL_PTR(conv_state_in);
    GDR_REQUIRE_PTR(dyq);
    GDR_REQUIRE_PTR(dyk);
    GDR_REQUIRE_PTR(dyv);
    GDR_OPTIONAL_PTR(dconv_state_out);
    GDR_REQUIRE_PTR(dxq);
    GDR_REQUIRE_PTR(dxk);
    GDR_REQUIRE_PTR(dxv);
    GDR_REQUIRE_PTR(dwq);
    GDR_REQUIRE_PTR(dwk);
    GDR_REQUIRE_PTR(dwv);
    GDR_OPTIONAL_PTR(dbq);
    GDR_OPTIONAL_PTR(dbk);
    GDR_OPTIONAL_PTR(dbv);
    GDR_OPTIONAL_PTR(dconv_state_in);
    const size_t need = prologue_bwd_workspace(H, dk, dv, K);
    if (workspace == nullptr || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", fn, workspace_bytes, need);
    if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: workspace is not 16-byte aligned", fn);
    PrologueBwdArgs a{};
    a.B = B; a.T = T; a.H = H; a.dk = dk; a.dv = dv; a.K = K;
    a.x[0] = xq; a.x[1] = xk; a.x[2] = xv;
    a.w[0] = wq; a.w[1] = wk; a.w[2] = wv;
    a.bias[0] = bq; a.bias[1] = bk; a.bias[2] = bv;
    a.state_in = K > 1 ? conv_state_in : nullptr;
    a.eps = eps;
    a.dy[0] = dyq; a.dy[1] = dyk; a.dy[2] = dyv;
    a.dstate_out = K > 1 ? dconv_state_out : nullptr;
    a.dx[0] = dxq; a.dx[1] = dxk; a.dx[2] = dxv;
    a.dstate_in = K > 1 ? dconv_state_in : nullptr;
    a.partial = static_cast<float *>(workspace);
    float *const dw[3] = {dwq, dwk, dwv};
    float *const db[3] = {dbq, dbk, dbv};
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    cudaError_t e = dt == GDR_F32 ? launch_prologue_bwd<float>(a, dw, db, s)
                                  : launch_prologue_bwd<__nv_bfloat16>(a, dw, db, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

gdr_status gdr_block_epilogue(int B, int T, int H, int dv, gdr_dtype dt, const void *o, const void *g,
                              const float *weight, float eps, void *y, gdr_stream_t stream) {
    const char *fn = "gdr_block_epilogue";
    gdr_status st = check_dims(fn, B, T, H, 64, dv, dt);
    if (st != GDR_OK) return st;
    if (!(eps >= 0.f) || eps > 1e30f) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: eps=%g", fn, (double)eps);
    GDR_REQUIRE_PTR(o);
    GDR_OPTIONAL_PTR(g);
    GDR_REQUIRE_PTR(weight);
    GDR_REQUIRE_PTR(y);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long rows = (long long)B * T * H;
    cudaError_t e = dt == GDR_F32 ? launch_epilogue<float>(rows, dv, o, g, weight, eps, y, s)
                                  : launch_epilogue<__nv_bfloat16>(rows, dv, o, g, weight, eps, y, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

size_t gdr_block_epilogue_bwd_workspace_bytes(int dv) {
    return (dv == 64 || dv == 128) ? (size_t)kEpiBwdMaxBlocks * dv * sizeof(float) : 0;
}

gdr_status gdr_block_epilogue_bwd(int B, int T, int H, int dv, gdr_dtype dt, const void *o, const void *g,
                                  const float *weight, float eps, const void *dy, void *dO, void *dg,
                                  float *dweight, void *workspace, size_t workspace_bytes, gdr_stream_t stream) {
    const char *fn = "gdr_block_epilogue_bwd";
    gdr_status st = check_dims(fn, B, T, H, 64, dv, dt);
    if (st != GDR_OK) return st;
    if (!(eps >= 0.f) || eps > 1e30f) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: eps=%g", fn, (double)eps);
    GDR_REQUIRE_PTR(o);
    GDR_OPTIONAL_PTR(g);
    GDR_REQUIRE_PTR(weight);
    GDR_REQUIRE_PTR(dy);
    GDR_REQUIRE_PTR(dO);
    GDR_REQUIRE_PTR(dweight);
    if ((g == nullptr) != (dg == nullptr))
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: g and dg must both be given or both NULL", fn);
    GDR_OPTIONAL_PTR(dg);
    const size_t need = gdr_block_epilogue_bwd_workspace_bytes(dv);
    if (workspace == nullptr || workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "%s: workspace %zu bytes, need %zu", fn, workspace_bytes, need);
    if (!aligned16(workspace)) return fail(GDR_ERR_INVALID_ARGUMENT, "%s: workspace is not 16-byte aligned", fn);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    const long long rows = (long long)B * T * H;
    float *partial = static_cast<float *>(workspace);
    cudaError_t e = dt == GDR_F32
                        ? launch_epilogue_bwd<float>(rows, dv, o, g, dy, weight, eps, dO, dg, dweight, partial, s)
                        : launch_epilogue_bwd<__nv_bfloat16>(rows, dv, o, g, dy, weight, eps, dO, dg, dweight, partial, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

size_t gdr_seg_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt) {
    if (B < 1 || T < 1 || H < 1 || (dk != 64 && dk != 128) || (dv != 64 && dv != 128) ||
        (dt != GDR_F32 && dt != GDR_BF16))
        return 0;
    const size_t es = dt == GDR_F32 ? 4 : 2;
    const size_t zero_v = ((size_t)B * T * H * dk * es + 255) & ~(size_t)255;
    return zero_v + (size_t)B * H * dk * dk * 4;
}

gdr_status gdr_seg_fwd(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *q, const void *k,
                       const void *v, const float *log_alpha, const float *beta, void *o0, void *qt, float *N,
                       float *M, void *workspace, size_t workspace_bytes, gdr_stream_t stream) {
    const char *fn = "gdr_seg_fwd";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(beta);
    GDR_REQUIRE_PTR(o0);
    GDR_REQUIRE_PTR(qt);
    GDR_REQUIRE_PTR(N);
    GDR_REQUIRE_PTR(M);
    GDR_REQUIRE_PTR(workspace);
    const size_t need = gdr_seg_fwd_workspace_bytes(B, T, H, dk, dv, dt);
    if (workspace_bytes < need)
        return fail(GDR_ERR_WORKSPACE, "%s: workspace of %zu bytes needed, %zu given", fn, need, workspace_bytes);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    std::lock_guard<std::mutex> lock(g_seg_mu);
    SegAux *auxp = nullptr;
    cudaError_t e = seg_aux(&auxp);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    SegAux &aux = *auxp;
    e = cudaEventRecord(aux.fork, s);
    if (e == cudaSuccess) e = cudaStreamWaitEvent(aux.stream, aux.fork, 0);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    // pass 1 (caller's stream): from S_in = 0 -> o(0) and N
    st = gdr_fwd(B, T, H, dk, dv, dt, q, k, v, log_alpha, beta, nullptr, o0, N, nullptr, 0, stream);
    // pass 2 (auxiliary stream): v = 0 from S_in = I (dv = dk) -> q~ and M
    const size_t es = dt == GDR_F32 ? 4 : 2;
    const size_t zero_v = ((size_t)B * T * H * dk * es + 255) & ~(size_t)255;
    uint8_t *ws = static_cast<uint8_t *>(workspace);
    float *eye = reinterpret_cast<float *>(ws + zero_v);
    gdr_status st2 = GDR_OK;
    e = cudaMemsetAsync(ws, 0, (size_t)B * T * H * dk * es, aux.stream);
    if (e == cudaSuccess) e = launch_seg_identity(eye, B * H, dk, aux.stream);
    if (e == cudaSuccess)
        st2 = gdr_fwd(B, T, H, dk, dk, dt, q, k, ws, log_alpha, beta, eye, qt, M, nullptr, 0,
                      reinterpret_cast<gdr_stream_t>(aux.stream));
    // join (always, so the caller's stream never runs ahead of pass 2)
    cudaError_t ej = cudaEventRecord(aux.join, aux.stream);
    if (ej == cudaSuccess) ej = cudaStreamWaitEvent(s, aux.join, 0);
    if (st != GDR_OK) return st;
    if (e != cudaSuccess) return cuda_fail(e, fn);
    if (st2 != GDR_OK) return st2;
    if (ej != cudaSuccess) return cuda_fail(ej, fn);
    return GDR_OK;
}

gdr_status gdr_seg_combine(int R, int r, int B, int H, int dk, int dv, const float *M, const float *N,
                           const float *S0, float *S_in, float *S_T, gdr_stream_t stream) {
    const char *fn = "gdr_seg_combine";
    gdr_status st = check_dims(fn, B, 1, H, dk, dv, GDR_F32);
    if (st != GDR_OK) return st;
    if (R < 1 || r < 0 || r >= R)
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: segment %d of %d", fn, r, R);
    if (S_in == nullptr && S_T == nullptr)
        return fail(GDR_ERR_INVALID_ARGUMENT, "%s: S_in and S_T are both NULL", fn);
    GDR_REQUIRE_PTR(M);
    GDR_REQUIRE_PTR(N);
    GDR_OPTIONAL_PTR(S0);
    GDR_OPTIONAL_PTR(S_in);
    GDR_OPTIONAL_PTR(S_T);
    cudaError_t e = launch_seg_combine(R, r, B * H, dk, dv, M, N, S0, S_in, S_T, reinterpret_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

gdr_status gdr_seg_fixup(int B, int T, int H, int dk, int dv, gdr_dtype dt, const void *qt, const float *S_in,
                         void *o, gdr_stream_t stream) {
    const char *fn = "gdr_seg_fixup";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(qt);
    GDR_REQUIRE_PTR(S_in);
    GDR_REQUIRE_PTR(o);
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    // bf16 with dk = dv = 128 on the tensor cores (GDR_SEG_FIXUP=simt selects
    // the CUDA-core kernel, used to cross-check it)
    const char *sel = getenv("GDR_SEG_FIXUP");
    const bool tc = dt == GDR_BF16 && dk == 128 && dv == 128 && !(sel && strcmp(sel, "simt") == 0);
    cudaError_t e = tc ? launch_seg_fixup_tc(B, T, H, qt, S_in, o, s)
                  : dt == GDR_F32 ? launch_seg_fixup<float>(B, T, H, dk, dv, qt, S_in, o, s)
                                  : launch_seg_fixup<__nv_bfloat16>(B, T, H, dk, dv, qt, S_in, o, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}

}  // extern "C"

// ---- gdr_bwd_noalloc: backward with library-owned static scratch -------------
// For callers that cannot allocate device memory: the scratch is this
// file-scope device array (64 MiB on every GPU that loads the library).  In
// host code `g_bwd_static_scratch` only names the symbol; its device address
// comes from cudaGetSymbolAddress, resolved once per device.
namespace {
constexpr size_t kBwdStaticScratchBytes = (size_t)64 << 20;
constexpr int kMaxDevices = 64;
std::mutex g_scratch_mu;
void *g_scratch_ptr[kMaxDevices] = {};
}  // namespace
static __device__ __align__(256) unsigned char g_bwd_static_scratch[kBwdStaticScratchBytes];

extern "C" gdr_status gdr_bwd_noalloc(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                                      const void *q, const void *k, const void *v,
                                      const float *log_alpha, const float *beta, const float *S0,
                                      const void *dO, const float *dS_T, void *dq, void *dk_out,
                                      void *dv_out, float *dlog_alpha, float *dbeta, float *dS0,
                                      gdr_stream_t stream) {
    const char *fn = "gdr_bwd_noalloc";
    gdr_status st = check_dims(fn, B, T, H, dk, dv, dt);
    if (st != GDR_OK) return st;
    GDR_REQUIRE_PTR(q);
    GDR_REQUIRE_PTR(k);
    GDR_REQUIRE_PTR(v);
    GDR_REQUIRE_PTR(log_alpha);
    GDR_REQUIRE_PTR(beta);
    GDR_REQUIRE_PTR(dO);
    GDR_REQUIRE_PTR(dq);
    GDR_REQUIRE_PTR(dk_out);
    GDR_REQUIRE_PTR(dv_out);
    GDR_REQUIRE_PTR(dlog_alpha);
    GDR_REQUIRE_PTR(dbeta);
    GDR_OPTIONAL_PTR(S0);
    GDR_OPTIONAL_PTR(dS_T);
    GDR_OPTIONAL_PTR(dS0);
    const size_t need = bwd_scratch_bytes(B, T, H, dk, dv, dt);
    if (need > kBwdStaticScratchBytes)
        return fail(GDR_ERR_WORKSPACE,
                    "%s: this problem needs %zu bytes of scratch; the static scratch holds %zu "
                    "(use gdr_bwd with a caller workspace)",
                    fn, need, kBwdStaticScratchBytes);
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return cuda_fail(e, "gdr_bwd_noalloc: cudaGetDevice");
    if (dev < 0 || dev >= kMaxDevices)
        return fail(GDR_ERR_UNSUPPORTED, "%s: device ordinal %d out of range", fn, dev);
    void *scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mu);
        if (g_scratch_ptr[dev] == nullptr) {
            e = cudaGetSymbolAddress(&g_scratch_ptr[dev], g_bwd_static_scratch);
            if (e != cudaSuccess) {
                g_scratch_ptr[dev] = nullptr;
                return cuda_fail(e, "gdr_bwd_noalloc: cudaGetSymbolAddress");
            }
        }
        scratch = g_scratch_ptr[dev];
    }
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    e = run_bwd(B, T, H, dk, dv, dt, q, k, v, log_alpha, beta, S0, dO, dS_T, dq, dk_out, dv_out, dlog_alpha,
                dbeta, dS0, scratch, s);
    if (e != cudaSuccess) return cuda_fail(e, fn);
    return GDR_OK;
}
