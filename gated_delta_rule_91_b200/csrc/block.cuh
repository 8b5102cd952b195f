// block.cuh -- the Gated DeltaNet block's pre- and post-processing around the
// gated delta rule, each one HBM pass:
//
//   prologue  q, k: ShortConv -> SiLU -> L2 normalisation per (token, head)
//             v   : ShortConv -> SiLU
//   epilogue  y = RMSNorm(o) * weight * SiLU(g)
//
// Source: the Gated DeltaNet review (meaningful96.github.io/nr/GDN), section
// 3.8 "Gated DeltaNet Block" (the q/k/v paths and the normalised, gated
// output), and the block-design paragraph of "Gated DeltaNet-2: Decoupling
// Erase and Write in Linear Attention" (short convolution + SiLU, q/k L2 norm,
// RMSNorm and a SiLU output gate).  The pages fix no widths or epsilons; the
// convolution is depthwise and causal, of width K (1..8), in the
// cross-correlation convention of a framework Conv1d:
//     z[t, c] = bias[c] + sum_{j<K} w[c, j] x[t-K+1+j, c],
// with the tokens before the first read from a carried conv state.
//
// Both kernels are bandwidth-bound streams: one warp owns a run of tokens of
// one (stream, batch, head) and each lane owns d/32 channels of it, so a row
// is one coalesced warp access; the causal window lives in registers and the
// per-head norms are warp-shuffle reductions.  Grids are sized to the SM
// count times the resident blocks and walk the units with a stride.
#pragma once

#include <algorithm>

#include "common.cuh"
#include "sm100.cuh"

namespace gdr {

constexpr int kBlkThreads = 256;  // 8 warps
constexpr int kConvMax = 8;       // widest ShortConv handled
constexpr int kPrologueRun = 64;  // tokens per prologue work unit
constexpr int kEpilogueRows = 8;    // rows per epilogue work unit

// ---- CPL consecutive elements per lane ---------------------------------------
template <int CPL> __device__ __forceinline__ void ld_row(const float *p, float *o) {
    if constexpr (CPL == 4) {
        float4 a = *reinterpret_cast<const float4 *>(p);
        o[0] = a.x; o[1] = a.y; o[2] = a.z; o[3] = a.w;
    } else {
        float2 a = *reinterpret_cast<const float2 *>(p);
        o[0] = a.x; o[1] = a.y;
    }
}
template <int CPL> __device__ __forceinline__ void ld_row(const __nv_bfloat16 *p, float *o) {
    if constexpr (CPL == 4) {
        uint2 raw = *reinterpret_cast<const uint2 *>(p);
        float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
        float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
        o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
    } else {
        uint32_t raw = *reinterpret_cast<const uint32_t *>(p);
        float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw));
        o[0] = a.x; o[1] = a.y;
    }
}
template <int CPL> __device__ __forceinline__ void st_row(float *p, const float *v) {
    if constexpr (CPL == 4)
        *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
    else
        *reinterpret_cast<float2 *>(p) = make_float2(v[0], v[1]);
}
template <int CPL> __device__ __forceinline__ void st_row(__nv_bfloat16 *p, const float *v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]);
    if constexpr (CPL == 4) {
        __nv_bfloat162 b = __floats2bfloat162_rn(v[2], v[3]);
        uint2 raw;
        raw.x = *reinterpret_cast<uint32_t *>(&a);
        raw.y = *reinterpret_cast<uint32_t *>(&b);
        *reinterpret_cast<uint2 *>(p) = raw;
    } else {
        *reinterpret_cast<__nv_bfloat162 *>(p) = a;
    }
}

// A row slice kept packed in its storage type until it is used, so a batch of
// bf16 rows in flight costs half the registers of the converted floats.
template <typename Tio, int CPL> struct RawRow;
template <> struct RawRow<float, 4> { float4 v; };
template <> struct RawRow<float, 2> { float2 v; };
template <> struct RawRow<__nv_bfloat16, 4> { uint2 v; };
template <> struct RawRow<__nv_bfloat16, 2> { uint32_t v; };

template <typename Tio, int CPL> __device__ __forceinline__ RawRow<Tio, CPL> ld_raw(const Tio *p) {
    RawRow<Tio, CPL> r;
    r.v = *reinterpret_cast<const decltype(r.v) *>(p);
    return r;
}
__device__ __forceinline__ void unpack(const RawRow<float, 4> &r, float *o) {
    o[0] = r.v.x; o[1] = r.v.y; o[2] = r.v.z; o[3] = r.v.w;
}
__device__ __forceinline__ void unpack(const RawRow<float, 2> &r, float *o) { o[0] = r.v.x; o[1] = r.v.y; }
__device__ __forceinline__ void unpack(const RawRow<__nv_bfloat16, 4> &r, float *o) {
    uint2 raw = r.v;
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.x));
    float2 b = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw.y));
    o[0] = a.x; o[1] = a.y; o[2] = b.x; o[3] = b.y;
}
__device__ __forceinline__ void unpack(const RawRow<__nv_bfloat16, 2> &r, float *o) {
    uint32_t raw = r.v;
    float2 a = __bfloat1622float2(*reinterpret_cast<__nv_bfloat162 *>(&raw));
    o[0] = a.x; o[1] = a.y;
}

__device__ __forceinline__ float silu_f(float z) { return z / (1.f + __expf(-z)); }

// ---- prologue -------------------------------------------------------------------
struct PrologueArgs {
    int B, T, H, dk, dv, K;
    const void *x[3];    // projected q, k, v: [B, T, H, d_s]
    const float *w[3];   // [H*d_s, K]
    const float *bias[3];  // [H*d_s] or null
    const void *state_in;  // [B, K-1, H*(2dk+dv)] or null (zeros)
    void *state_out;       // same layout or null (not written); may equal state_in
    float eps;
    void *y[3];          // q, k, v outputs, [B, T, H, d_s]
};

// A unit is one (stream, batch, head) and a run of kPrologueRun tokens.  Its
// rows -- the K-1 tokens before the run, then the run -- are staged in shared
// memory: row r holds token t0 - (K-1) + r, so output token t0 + i reads rows
// i .. i+K-1.  Two stages: the next unit's bulk copies fly while this one is
// computed.
constexpr int kPrologueRows = kPrologueRun + kConvMax - 1;

struct PrologueUnit {
    int s, b, h, t0, len, d;
};

__device__ __forceinline__ PrologueUnit prologue_decode(const PrologueArgs &a, long long u) {
    const int runs = (a.T + kPrologueRun - 1) / kPrologueRun;
    const long long per_stream = (long long)a.B * a.H * runs;
    PrologueUnit p;
    p.s = (int)(u / per_stream);
    long long r = u - p.s * per_stream;
    const int run = (int)(r % runs);
    r /= runs;
    p.h = (int)(r % a.H);
    p.b = (int)(r / a.H);
    p.t0 = run * kPrologueRun;
    p.len = min(kPrologueRun, a.T - p.t0);
    p.d = p.s < 2 ? a.dk : a.dv;
    return p;
}

// Stream pointers by selects (a runtime index into the parameter block would
// copy it to local memory).
template <typename Tio> __device__ __forceinline__ const Tio *prologue_x(const PrologueArgs &a, int s) {
    return static_cast<const Tio *>(s == 0 ? a.x[0] : s == 1 ? a.x[1] : a.x[2]);
}

// Channel offset of stream s in the conv state.
__device__ __forceinline__ int prologue_state_col(const PrologueArgs &a, int s) {
    return s == 0 ? 0 : s == 1 ? a.H * a.dk : 2 * a.H * a.dk;
}

// Warp 0 stages unit p into `stage` (row bytes = d * sizeof(Tio), a multiple
// of 128): bulk copies for tokens read from x or the old conv state, plain
// zero stores for tokens before the start with no state.
template <typename Tio>
__device__ __forceinline__ void prologue_stage(const PrologueArgs &a, const PrologueUnit &p, uint8_t *stage,
                                               uint64_t *bar, int lane) {
    using namespace sm100;
    const int K = a.K, rows = p.len + K - 1;
    const uint32_t rb = (uint32_t)p.d * sizeof(Tio);
    const int first = p.t0 - (K - 1);  // token of row 0
    // bytes arriving by bulk copy
    int zero_rows = 0;
    if (first < 0 && a.state_in == nullptr) zero_rows = -first;
    if (lane == 0) mbar_expect_tx(bar, (uint32_t)(rows - zero_rows) * rb);
    __syncwarp();
    const Tio *x = prologue_x<Tio>(a, p.s);
    const int Ctot = a.H * (2 * a.dk + a.dv);
    for (int r = lane; r < rows; r += 32) {
        const int t = first + r;
        uint8_t *dst = stage + (size_t)r * rb;
        if (t >= 0) {
            bulk_load_g2s(dst, x + (((size_t)p.b * a.T + t) * a.H + p.h) * p.d, rb, bar);
        } else if (a.state_in) {
            const Tio *st = static_cast<const Tio *>(a.state_in) +
                            ((size_t)p.b * (K - 1) + (K - 1 + t)) * Ctot + prologue_state_col(a, p.s) + p.h * p.d;
            bulk_load_g2s(dst, st, rb, bar);
        } else {
            for (uint32_t o = 0; o < rb; o += 16) *reinterpret_cast<uint4 *>(dst + o) = make_uint4(0, 0, 0, 0);
        }
    }
}

// Output rows of a staged unit: warp w takes rows w, w+8, ...; lane owns
// CPL = d/32 channels.  KW (4 or 8) is the register window, K <= KW.
template <typename Tio, int CPL, int KW>
__device__ __forceinline__ void prologue_compute(const PrologueArgs &a, const PrologueUnit &p, const uint8_t *stage,
                                                 int warp, int lane) {
    constexpr int D = CPL * 32;
    const int K = a.K;
    const int c0 = p.h * D + lane * CPL;  // first channel of this lane in the stream
    const float *wsel = p.s == 0 ? a.w[0] : p.s == 1 ? a.w[1] : a.w[2];
    const float *bsel = p.s == 0 ? a.bias[0] : p.s == 1 ? a.bias[1] : a.bias[2];
    Tio *y = static_cast<Tio *>(p.s == 0 ? a.y[0] : p.s == 1 ? a.y[1] : a.y[2]);
    float wt[CPL][KW], bias[CPL];  // wt[c][j] multiplies row i + j
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
#pragma unroll
        for (int j = 0; j < KW; ++j) wt[c][j] = j < K ? __ldg(wsel + (size_t)(c0 + c) * K + j) : 0.f;
        bias[c] = bsel ? __ldg(bsel + c0 + c) : 0.f;
    }
    const Tio *sm = reinterpret_cast<const Tio *>(stage) + lane * CPL;
    const bool l2 = p.s < 2;
#pragma unroll 1
    for (int i = warp; i < p.len; i += kBlkThreads / 32) {
        float acc[CPL];
#pragma unroll
        for (int c = 0; c < CPL; ++c) acc[c] = bias[c];
#pragma unroll
        for (int j = 0; j < KW; ++j) {
            if (j < K) {
                float xv[CPL];
                ld_row<CPL>(sm + (size_t)(i + j) * D, xv);
#pragma unroll
                for (int c = 0; c < CPL; ++c) acc[c] = fmaf(wt[c][j], xv[c], acc[c]);
            }
        }
        float ss = 0.f;
#pragma unroll
        for (int c = 0; c < CPL; ++c) {
            acc[c] = silu_f(acc[c]);
            ss = fmaf(acc[c], acc[c], ss);
        }
        if (l2) {
            const float inv = rsqrtf(warp_sum(ss, 32) + a.eps);
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[c] *= inv;
        }
        st_row<CPL>(y + (((size_t)p.b * a.T + p.t0 + i) * a.H) * D + c0, acc);
    }
}

// The carried state of (stream, batch, head): the last K-1 inputs.  Written by
// the run-0 unit after its stage (which holds the old state rows) is complete,
// so an in-place state is safe: no other unit reads the old state.
template <typename Tio, int CPL>
__device__ __forceinline__ void prologue_state_out(const PrologueArgs &a, const PrologueUnit &p,
                                                   const uint8_t *stage, int warp, int lane) {
    constexpr int D = CPL * 32;
    const int K = a.K, Ctot = a.H * (2 * a.dk + a.dv);
    const Tio *sm = reinterpret_cast<const Tio *>(stage) + lane * CPL;
    const Tio *x = prologue_x<Tio>(a, p.s);
    Tio *so = static_cast<Tio *>(a.state_out) + (size_t)p.b * (K - 1) * Ctot + prologue_state_col(a, p.s) + p.h * D +
              lane * CPL;
    for (int j = warp; j < K - 1; j += kBlkThreads / 32) {
        const int t = a.T - (K - 1) + j;  // token held by state row j
        float v[CPL];
        if (t < p.len)  // staged: row t + K - 1 (t >= -(K-1) always)
            ld_row<CPL>(sm + (size_t)(t + K - 1) * D, v);
        else
            ld_row<CPL>(x + (((size_t)p.b * a.T + t) * a.H + p.h) * D + lane * CPL, v);
        st_row<CPL>(so + (size_t)j * Ctot, v);
    }
}

template <typename Tio, int CPLQK, int CPLV, int KW>
__global__ void __launch_bounds__(kBlkThreads) gdr_prologue_kernel(const PrologueArgs a, int stage_bytes) {
    using namespace sm100;
    extern __shared__ __align__(128) uint8_t blk_smem[];
    uint8_t *smem = blk_smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + 2 * stage_bytes);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long units = 3LL * a.B * a.H * ((a.T + kPrologueRun - 1) / kPrologueRun);
    if (threadIdx.x == 0) {
        mbar_init(&bars[0], 1);
        mbar_init(&bars[1], 1);
        fence_mbar_init();
    }
    __syncthreads();
    long long u = blockIdx.x;
    if (u < units && warp == 0) prologue_stage<Tio>(a, prologue_decode(a, u), smem, &bars[0], lane);
    __syncthreads();  // zero-filled rows are plain stores: publish them to all warps
#pragma unroll 1
    for (int k = 0; u < units; ++k, u += gridDim.x) {
        const int st = k & 1;
        const PrologueUnit p = prologue_decode(a, u);
        // stage the next unit into the other buffer (its readers finished at
        // the barrier that ended the previous iteration)
        const long long un = u + gridDim.x;
        if (un < units && warp == 0) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            prologue_stage<Tio>(a, prologue_decode(a, un), smem + (st ^ 1) * stage_bytes, &bars[st ^ 1], lane);
        }
        if (!mbar_wait(&bars[st], (uint32_t)(k >> 1) & 1u)) {
            record_status(GDR_ERR_TIMEOUT);
            // let the copies already issued for the next unit land before the
            // block exits
            if (un < units) mbar_wait(&bars[st ^ 1], (uint32_t)((k + 1) >> 1) & 1u, 100000000ull);
            return;
        }
        const uint8_t *stage = smem + st * stage_bytes;
        if (p.s < 2)
            prologue_compute<Tio, CPLQK, KW>(a, p, stage, warp, lane);
        else
            prologue_compute<Tio, CPLV, KW>(a, p, stage, warp, lane);
        if (p.t0 == 0 && a.state_out != nullptr) {
            if (p.s < 2)
                prologue_state_out<Tio, CPLQK>(a, p, stage, warp, lane);
            else
                prologue_state_out<Tio, CPLV>(a, p, stage, warp, lane);
        }
        __syncthreads();
    }
}

// ---- epilogue ---------------------------------------------------------------------
// y = o / sqrt(mean(o^2) + eps) * weight * SiLU(g) per row of dv channels;
// g == nullptr leaves out the gate.  Rows are the B*T*H (token, head) pairs.
template <typename Tio, int CPL>
__global__ void __launch_bounds__(kBlkThreads)
    gdr_epilogue_kernel(long long rows, const Tio *__restrict__ o, const Tio *__restrict__ g,
                        const float *__restrict__ weight, float eps, Tio *__restrict__ y) {
    constexpr int D = CPL * 32;
    const int lane = threadIdx.x & 31;
    float wl[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) wl[c] = __ldg(weight + lane * CPL + c);
    const long long units = (rows + kEpilogueRows - 1) / kEpilogueRows;
    const long long nw = (long long)gridDim.x * (kBlkThreads / 32);
#pragma unroll 1
    for (long long u = (blockIdx.x * (long long)kBlkThreads + threadIdx.x) >> 5; u < units; u += nw) {
        const long long r0 = u * kEpilogueRows;
        const int n = (int)min((long long)kEpilogueRows, rows - r0);
        const size_t base = (size_t)r0 * D + lane * CPL;
        RawRow<Tio, CPL> orow[kEpilogueRows], grow[kEpilogueRows];
#pragma unroll
        for (int i = 0; i < kEpilogueRows; ++i) {
            if (i < n) {
                orow[i] = ld_raw<Tio, CPL>(o + base + (size_t)i * D);
                if (g) grow[i] = ld_raw<Tio, CPL>(g + base + (size_t)i * D);
            }
        }
#pragma unroll
        for (int i = 0; i < kEpilogueRows; ++i) {
            if (i >= n) break;
            float ov[CPL], gv[CPL], ss = 0.f;
            unpack(orow[i], ov);
            if (g) unpack(grow[i], gv);
#pragma unroll
            for (int c = 0; c < CPL; ++c) ss = fmaf(ov[c], ov[c], ss);
            const float inv = rsqrtf(warp_sum(ss, 32) * (1.f / D) + eps);
            float out[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) out[c] = ov[c] * inv * wl[c] * (g ? silu_f(gv[c]) : 1.f);
            st_row<CPL>(y + base + (size_t)i * D, out);
        }
    }
}

// Grid = SMs x resident blocks of the kernel (capped by the work), so the
// stride loop covers the units in whole waves.
// (One cached figure per kernel instantiation: the library runs on B200s only.)
template <typename Kern> inline int resident_grid(Kern kernel, long long warps_needed, int smem = 0) {
    static int per_sm = 0, sms = 0;
    if (per_sm == 0) {
        int dev = 0, nb = 0, ns = 0;
        if (cudaGetDevice(&dev) != cudaSuccess ||
            cudaDeviceGetAttribute(&ns, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
            cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, kBlkThreads, smem) != cudaSuccess)
            return 0;
        sms = ns;
        per_sm = nb > 0 ? nb : 1;
    }
    const long long blocks = (warps_needed + kBlkThreads / 32 - 1) / (kBlkThreads / 32);
    return (int)std::min<long long>(blocks, (long long)sms * per_sm);
}

template <typename Tio, int CPLQK, int CPLV>
inline cudaError_t launch_prologue_t(const PrologueArgs &a, cudaStream_t stream) {
    auto kern = a.K <= 4 ? gdr_prologue_kernel<Tio, CPLQK, CPLV, 4> : gdr_prologue_kernel<Tio, CPLQK, CPLV, kConvMax>;
    const int stage_bytes = kPrologueRows * 32 * (CPLQK > CPLV ? CPLQK : CPLV) * (int)sizeof(Tio);
    const int smem = 2 * stage_bytes + 16;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const long long units = 3LL * a.B * a.H * ((a.T + kPrologueRun - 1) / kPrologueRun);
    const int grid = resident_grid(kern, units * (kBlkThreads / 32), smem);
    if (grid <= 0) return cudaErrorInvalidConfiguration;
    kern<<<grid, kBlkThreads, smem, stream>>>(a, stage_bytes);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

template <typename Tio>
inline cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream) {
    if (a.dk == 128 && a.dv == 128) return launch_prologue_t<Tio, 4, 4>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_prologue_t<Tio, 4, 2>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_prologue_t<Tio, 2, 4>(a, stream);
    return launch_prologue_t<Tio, 2, 2>(a, stream);
}

template <typename Tio>
inline cudaError_t launch_epilogue(long long rows, int dv, const void *o, const void *g, const float *weight,
                                   float eps, void *y, cudaStream_t stream) {
    auto run = [&](auto kern) -> cudaError_t {
        const int grid = resident_grid(kern, (rows + kEpilogueRows - 1) / kEpilogueRows);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        kern<<<grid, kBlkThreads, 0, stream>>>(rows, static_cast<const Tio *>(o), static_cast<const Tio *>(g), weight,
                                               eps, static_cast<Tio *>(y));
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cudaGetLastError();
    };
    return dv == 128 ? run(gdr_epilogue_kernel<Tio, 4>) : run(gdr_epilogue_kernel<Tio, 2>);
}

}  // namespace gdr
