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
#include "fwd_tc.cuh"  // encode_tiled_fn

namespace gdr {

constexpr int kBlkThreads = 256;  // 8 warps
constexpr int kConvMax = 8;       // widest ShortConv handled
constexpr int kPrologueRun = 128;  // tokens per prologue work unit

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

// Special-function-unit approximations with denormals flushed (ex2.approx,
// rcp.approx, rsqrt.approx of the PTX ISA).
__device__ __forceinline__ float ex2_ftz(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rcp_ftz(float x) {
    float y;
    asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
__device__ __forceinline__ float rsqrt_ftz(float x) {
    float y;
    asm("rsqrt.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}
// SiLU(z) = z / (1 + e^-z), with e^-z = 2^(-z log2 e).  For z -> -inf the
// denominator overflows to +inf, its reciprocal is 0 and the result -0, the
// limit; for z -> +inf the result is z.
constexpr float kLog2e = 1.4426950408889634f;
__device__ __forceinline__ float silu_f(float z) { return z * rcp_ftz(1.f + ex2_ftz(-kLog2e * z)); }

// Packed fp32 pair arithmetic (fma.rn.f32x2 / mul.rn.f32x2): one instruction
// for two lanes' worth of FMAs, each rounded as the scalar one.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rc, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mov.b64 rc, {%6, %7};\n fma.rn.f32x2 rd, ra, rb, rc;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}
__device__ __forceinline__ float2 fmul2(float2 a, float2 b) {
    float2 d;
    asm("{\n .reg .b64 ra, rb, rd;\n mov.b64 ra, {%2, %3};\n mov.b64 rb, {%4, %5};\n"
        " mul.rn.f32x2 rd, ra, rb;\n mov.b64 {%0, %1}, rd;\n}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

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

// Work split.  A block owns one (stream, head) pair -- its conv taps and
// biases stay in registers -- and walks the (batch, run) units of that pair
// with a stride; unit = kPrologueRun tokens of one batch.  The grid is the
// 3H pairs times G blocks each; blocks with the same index on neighbouring
// heads read the same tokens at about the same time (whole HBM rows).
//
// A unit's rows -- the K-1 tokens before the run, then the run -- arrive by
// one tiled TMA load into a ring stage: row r holds token t0 - (K-1) + r, so
// output token t0 + i reads rows i .. i+K-1.  Tokens before 0 or past T read
// as zero; rows from a carried conv state are patched in after the load.
constexpr int kPrologueRows = kPrologueRun + kConvMax - 1;
constexpr int kBlkStages = 3;  // bulk-copy ring depth of the staged kernels
constexpr int kProStages = 3;  // ring depth of the prologue

// After a wait gave up at unit k (stage st): wait, with a short bound, for the
// copies already issued into the other stages so that none lands after the
// block has exited.
template <int NS>
__device__ __forceinline__ void blk_drain(uint64_t *bars, int st, int k, long long u, long long units,
                                          long long stride) {
    for (int m = 1; m < NS; ++m)
        if (u + (long long)m * stride < units)
            sm100::mbar_wait(&bars[(st + m) % NS], (uint32_t)((k + m) / NS) & 1u, 100000000ull);
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

__device__ __forceinline__ void store8(float *p, const float *v) {
    reinterpret_cast<float4 *>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4 *>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}
__device__ __forceinline__ void store8(__nv_bfloat16 *p, const float *v) {
    uint4 raw;
    __nv_bfloat162 h0 = __floats2bfloat162_rn(v[0], v[1]), h1 = __floats2bfloat162_rn(v[2], v[3]);
    __nv_bfloat162 h2 = __floats2bfloat162_rn(v[4], v[5]), h3 = __floats2bfloat162_rn(v[6], v[7]);
    raw.x = *reinterpret_cast<uint32_t *>(&h0);
    raw.y = *reinterpret_cast<uint32_t *>(&h1);
    raw.z = *reinterpret_cast<uint32_t *>(&h2);
    raw.w = *reinterpret_cast<uint32_t *>(&h3);
    *reinterpret_cast<uint4 *>(p) = raw;
}

// The block's part of the prologue for stream s, head h (D channels).  A lane
// owns 8 channels and a group of D/8 lanes one row (the L2 norm is a
// reduction inside the group); the groups of the block take consecutive row
// blocks of the run and slide a K-row window down theirs, so each staged row
// is read about once.  The window holds KW (4 or 8) rows with the taps
// right-aligned: win[m] is row i + K - KW + m and taps m < KW - K are zero.
// Every lane runs the same trip count (rows past the run are computed from
// in-bounds stage memory and not stored), so the group shuffles always have
// the full warp.
template <typename Tio, int D, int KW>
__device__ __forceinline__ void prologue_block(const PrologueArgs &a, const CUtensorMap *map, int s, int h, int idx,
                                               int G, uint8_t *smem, int stage_bytes, uint64_t *bars) {
    using namespace sm100;
    constexpr int CPL = 8, LPR = D / CPL, GPW = 32 / LPR;
    constexpr int RPG = kPrologueRun / ((kBlkThreads / 32) * GPW);  // rows per group
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = a.K, T = a.T;
    const int runs = (T + kPrologueRun - 1) / kPrologueRun;
    const int units = a.B * runs;  // (batch, run) units of this pair; B*T*H*d < 2^31 on the host
    const int sl = lane % LPR, i0 = (warp * GPW + lane / LPR) * RPG;
    const int c0 = h * D + sl * CPL;  // first channel of this lane in the stream
    const uint32_t box_bytes = (uint32_t)(kPrologueRun + K - 1) * D * (uint32_t)sizeof(Tio);

    // taps (right-aligned in the window) and biases of this lane's channels
    const float *wsel = s == 0 ? a.w[0] : s == 1 ? a.w[1] : a.w[2];
    const float *bsel = s == 0 ? a.bias[0] : s == 1 ? a.bias[1] : a.bias[2];
    float wt[CPL][KW], bias[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
#pragma unroll
        for (int m = 0; m < KW; ++m) {
            const int j = m - (KW - K);  // tap index
            wt[c][m] = j >= 0 ? __ldg(wsel + (size_t)(c0 + c) * K + j) : 0.f;
        }
        bias[c] = bsel ? __ldg(bsel + c0 + c) : 0.f;
    }

    // the ring: unit k of this block is (batch, run) idx + k*G, in stage
    // k % kProStages with phase parity (k / kProStages) & 1
    auto issue = [&](int k, int sidx) {  // one thread
        const int j = idx + k * G, b = j / runs, t0 = (j % runs) * kPrologueRun;
        mbar_expect_tx(&bars[sidx], box_bytes);
        tma_load_4d(smem + sidx * stage_bytes, map, &bars[sidx], 0, h, t0 - (K - 1), b);
    };
    if (threadIdx.x == 0)
        for (int k = 0; k < kProStages - 1; ++k)
            if (idx + k * G < units) issue(k, k);
    const bool l2 = s < 2;
    const size_t ystride = (size_t)a.H * D;
    Tio *ybase = static_cast<Tio *>(s == 0 ? a.y[0] : s == 1 ? a.y[1] : a.y[2]);
    int st = 0;
#pragma unroll 1
    for (int k = 0;; ++k) {
        const int j = idx + k * G;
        if (j >= units) break;
        const int b = j / runs, t0 = (j % runs) * kPrologueRun, len = min(kPrologueRun, T - t0);
        // stage unit k + kProStages - 1 into the slot unit k - 1 used (its
        // readers finished at the barrier that ended the previous iteration)
        if (threadIdx.x == 0 && j + (kProStages - 1) * G < units) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(k + kProStages - 1, st == 0 ? kProStages - 1 : st - 1);
        }
        if (!mbar_wait(&bars[st], (uint32_t)(k / kProStages) & 1u)) {
            record_status(GDR_ERR_TIMEOUT);
            blk_drain<kProStages>(bars, st, k, j, units, G);
            return;
        }
        uint8_t *stage = smem + st * stage_bytes;
        const int Ctot = a.H * (2 * a.dk + a.dv);
        if (t0 == 0 && a.state_in != nullptr && K > 1) {
            // rows 0 .. K-2 (read as zero by the TMA) take the old state's rows
            constexpr int kPieces = D * (int)sizeof(Tio) / 16;
            for (int i = threadIdx.x; i < (K - 1) * kPieces; i += kBlkThreads) {
                const int r = i / kPieces, q = i % kPieces;
                const Tio *src = static_cast<const Tio *>(a.state_in) + ((size_t)b * (K - 1) + r) * Ctot +
                                 prologue_state_col(a, s) + h * D;
                reinterpret_cast<uint4 *>(stage + (size_t)r * D * sizeof(Tio))[q] =
                    reinterpret_cast<const uint4 *>(src)[q];
            }
            __syncthreads();
        }

        const Tio *sx = reinterpret_cast<const Tio *>(stage) + sl * CPL;
        float win[KW][CPL];
#pragma unroll
        for (int m = 0; m < KW - 1; ++m) {
            const int row = i0 + K - KW + m;
            if (row >= 0)
                load8(sx + row * D, win[m]);
            else
#pragma unroll
                for (int c = 0; c < CPL; ++c) win[m][c] = 0.f;
        }
        Tio *y = ybase + (((size_t)b * T + t0 + i0) * a.H) * D + c0;
        // batches of NB rows: conv + SiLU for each, then their norm
        // reductions interleaved (independent shuffle chains), then stores
        constexpr int NB = RPG < 4 ? RPG : 4;
#pragma unroll
        for (int r0 = 0; r0 < RPG; r0 += NB) {
            float acc[NB][CPL], ss[NB];
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                load8(sx + (i0 + r0 + q + K - 1) * D, win[KW - 1]);
                float2 ss2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int c = 0; c < CPL; c += 2) {  // channel pairs on the packed FMA
                    float2 z = make_float2(bias[c], bias[c + 1]);
#pragma unroll
                    for (int m = 0; m < KW; ++m)
                        z = ffma2(make_float2(wt[c][m], wt[c + 1][m]), make_float2(win[m][c], win[m][c + 1]), z);
                    acc[q][c] = silu_f(z.x);
                    acc[q][c + 1] = silu_f(z.y);
                    ss2 = ffma2(make_float2(acc[q][c], acc[q][c + 1]), make_float2(acc[q][c], acc[q][c + 1]), ss2);
                }
                ss[q] = ss2.x + ss2.y;
#pragma unroll
                for (int m = 0; m < KW - 1; ++m)
#pragma unroll
                    for (int c = 0; c < CPL; ++c) win[m][c] = win[m + 1][c];
            }
            if (l2) {
#pragma unroll
                for (int off = LPR / 2; off > 0; off >>= 1)
#pragma unroll
                    for (int q = 0; q < NB; ++q) ss[q] += __shfl_xor_sync(0xffffffffu, ss[q], off);
#pragma unroll
                for (int q = 0; q < NB; ++q) {
                    const float inv = rsqrt_ftz(ss[q] + a.eps);
#pragma unroll
                    for (int c = 0; c < CPL; c += 2) {
                        const float2 t = fmul2(make_float2(acc[q][c], acc[q][c + 1]), make_float2(inv, inv));
                        acc[q][c] = t.x;
                        acc[q][c + 1] = t.y;
                    }
                }
            }
#pragma unroll
            for (int q = 0; q < NB; ++q)
                if (i0 + r0 + q < len) store8(y + (r0 + q) * ystride, acc[q]);
        }

        // The carried state of (stream, batch, head): the last K-1 inputs,
        // written by the run-0 unit after its stage (holding the old state
        // rows) is complete, so an in-place state is safe: no other unit reads
        // the old state.
        if (t0 == 0 && a.state_out != nullptr && K > 1) {
            const Tio *x = prologue_x<Tio>(a, s);
            Tio *so = static_cast<Tio *>(a.state_out) + (size_t)b * (K - 1) * Ctot + prologue_state_col(a, s) + h * D;
            constexpr int kPieces = D * (int)sizeof(Tio) / 16;
            for (int i = threadIdx.x; i < (K - 1) * kPieces; i += kBlkThreads) {
                const int jr = i / kPieces, q = i % kPieces;
                const int t = T - (K - 1) + jr;  // token held by state row jr
                const uint4 *src = t < len ? reinterpret_cast<const uint4 *>(stage + (size_t)(t + K - 1) * D * sizeof(Tio))
                                           : reinterpret_cast<const uint4 *>(x + (((size_t)b * T + t) * a.H + h) * D);
                reinterpret_cast<uint4 *>(so + (size_t)jr * Ctot)[q] = src[q];
            }
        }
        __syncthreads();
        st = st == kProStages - 1 ? 0 : st + 1;
    }
}

template <typename Tio, int DQK, int DV, int KW>
__global__ void __launch_bounds__(kBlkThreads)
    gdr_prologue_kernel(const PrologueArgs a, int stage_bytes, const __grid_constant__ CUtensorMap tm_q,
                        const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v) {
    using namespace sm100;
    extern __shared__ __align__(128) uint8_t blk_smem[];
    uint8_t *smem = blk_smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kProStages * stage_bytes);
    const int P = 3 * a.H, pair = blockIdx.x % P, idx = blockIdx.x / P, G = gridDim.x / P;
    const int s = pair / a.H, h = pair % a.H;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kProStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    __syncthreads();
    if (s == 0)
        prologue_block<Tio, DQK, KW>(a, &tm_q, s, h, idx, G, smem, stage_bytes, bars);
    else if (s == 1)
        prologue_block<Tio, DQK, KW>(a, &tm_k, s, h, idx, G, smem, stage_bytes, bars);
    else
        prologue_block<Tio, DV, KW>(a, &tm_v, s, h, idx, G, smem, stage_bytes, bars);
}

// ---- prologue backward ----------------------------------------------------------
// Reverse mode of the prologue, per stream, for incoming dy (and optionally
// the gradient of the returned conv state):
//   recompute z = conv(x), u = SiLU(z), n = sqrt(sum_head u^2 + eps)
//   du = (dy - y (y . dy)) / n   with y = u / n   (q, k; du = dy for v)
//   dz = du sig(z) (1 + z (1 - sig(z)))
//   dx[s] = sum_j w[j] dz[s + K-1-j] (+ dstate_out where x[s] is carried out;
//           s < 0: dstate_in)
//   dw[c, j] = sum_t dz[t, c] x[t-K+1+j, c],   dbias[c] = sum_t dz[t, c].
// Same (stream, head) pair ownership as the forward.  A unit is 64 tokens
// [t0, t0+64); a block owns a contiguous range of the pair's (batch, run)
// units and walks it from the last to the first.  The stage holds x for
// tokens t0-(K-1) .. t0+63 and dy for t0 .. t0+63 (one tiled TMA load each,
// zero past T).  dx of the unit's last tokens needs dz of the K-1 tokens
// after it: those are the first rows of the unit walked just before, carried
// in shared memory (zero at the end of a batch; computed from global memory
// for the block's first unit).  Phase 1 (D/32 channels per lane, 8
// consecutive rows per warp) recomputes dz into a fp32 shared buffer and adds
// the rows into the lane's dw and dbias registers; phase 2 forms dx from a
// sliding window of dz rows.  At the end the block adds its warps' sums in
// warp order into one row of `partial`, and a second launch adds the G blocks
// of each pair in block order.
constexpr int kProBwdRun = 64;
constexpr int kProBwdStages = 2;
constexpr int kProBwdRowsPerWarp = kProBwdRun / (kBlkThreads / 32);  // 8 consecutive rows per warp
constexpr int kProBwdNB = 2;  // dz rows per step of phase 1
constexpr int kProBwdMaxG = 32;  // blocks per (stream, head) pair: the workspace bound

struct PrologueBwdArgs {
    int B, T, H, dk, dv, K;
    const void *x[3];
    const float *w[3];
    const float *bias[3];   // or null (zero)
    const void *state_in;   // [B, K-1, H*(2dk+dv)] or null (zeros)
    float eps;
    const void *dy[3];      // incoming gradients of q, k, v
    const void *dstate_out; // gradient of the returned conv state, or null
    void *dx[3];
    void *dstate_in;        // gradient of the carried-in state, or null (not written)
    float *partial;         // [3H*G][DMAX*(KW+1)]: per-block dw (slots 0..K-1) and dbias (slot KW)
    int partial_stride;     // DMAX*(KW+1)
};

template <typename Tio, int D, int KW>
__device__ __forceinline__ void prologue_bwd_block(const PrologueBwdArgs &a, const CUtensorMap *mx,
                                                   const CUtensorMap *mdy, int s, int h, int idx, int G,
                                                   uint8_t *smem, int stage_bytes, int xalloc, float *dzs,
                                                   uint64_t *bars) {
    using namespace sm100;
    // a lane owns CPL = D/32 channels as NP pairs: every elementwise step runs
    // on the packed fp32 pair instructions (each lane rounded as the scalar op)
    constexpr int CPL = D / 32, NP = CPL / 2, NW = kBlkThreads / 32;
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int K = a.K, T = a.T, H = a.H;
    const int runs = (T + kProBwdRun - 1) / kProBwdRun;
    const int units = a.B * runs;
    // this block's units, walked from the last to the first
    const int j_lo = (int)((long long)idx * units / G), j_hi = (int)((long long)(idx + 1) * units / G);
    const int n_my = j_hi - j_lo;
    const int c0 = h * D + lane * CPL;  // this lane's first channel in the stream
    const uint32_t xbox = (uint32_t)(kProBwdRun + K - 1) * D * (uint32_t)sizeof(Tio);
    const uint32_t dybox = (uint32_t)kProBwdRun * D * (uint32_t)sizeof(Tio);
    const int Ctot = H * (2 * a.dk + a.dv);
    const int col = s == 0 ? 0 : s == 1 ? H * a.dk : 2 * H * a.dk;  // stream's columns in the state

    const float *wsel = s == 0 ? a.w[0] : s == 1 ? a.w[1] : a.w[2];
    const float *bsel = s == 0 ? a.bias[0] : s == 1 ? a.bias[1] : a.bias[2];
    // taps right-aligned as in the forward: wt[p][m] holds tap m - (KW - K) of
    // the pair's two channels, and taps m < KW - K are zero; dwa[p][m] sums
    // the gradient of the same tap
    float2 wt[NP][KW], bias[NP], dwa[NP][KW], dba[NP];
#pragma unroll
    for (int p = 0; p < NP; ++p) {
#pragma unroll
        for (int m = 0; m < KW; ++m) {
            const int j = m - (KW - K);
            wt[p][m] = j >= 0 ? make_float2(__ldg(wsel + (size_t)(c0 + 2 * p) * K + j),
                                            __ldg(wsel + (size_t)(c0 + 2 * p + 1) * K + j))
                              : make_float2(0.f, 0.f);
            dwa[p][m] = make_float2(0.f, 0.f);
        }
        bias[p] = bsel ? make_float2(__ldg(bsel + c0 + 2 * p), __ldg(bsel + c0 + 2 * p + 1)) : make_float2(0.f, 0.f);
        dba[p] = make_float2(0.f, 0.f);
    }
    auto issue = [&](int k, int sidx) {  // one thread
        const int j = j_hi - 1 - k, b = j / runs, t0 = (j % runs) * kProBwdRun;
        uint8_t *stg = smem + sidx * stage_bytes;
        mbar_expect_tx(&bars[sidx], xbox + dybox);
        tma_load_4d(stg, mx, &bars[sidx], 0, h, t0 - (K - 1), b);
        tma_load_4d(stg + xalloc, mdy, &bars[sidx], 0, h, t0, b);
    };
    if (threadIdx.x == 0)
        for (int k = 0; k < kProBwdStages - 1; ++k)
            if (k < n_my) issue(k, k);
    const bool l2 = s < 2;
    const Tio *xg = static_cast<const Tio *>(s == 0 ? a.x[0] : s == 1 ? a.x[1] : a.x[2]);
    const Tio *dyg = static_cast<const Tio *>(s == 0 ? a.dy[0] : s == 1 ? a.dy[1] : a.dy[2]);
    const Tio *dso = static_cast<const Tio *>(a.dstate_out);
    Tio *dxb = static_cast<Tio *>(s == 0 ? a.dx[0] : s == 1 ? a.dx[1] : a.dx[2]);
    Tio *dsi = static_cast<Tio *>(a.dstate_in);
    const float2 one2 = make_float2(1.f, 1.f), mone2 = make_float2(-1.f, -1.f);
    const float2 ml2e2 = make_float2(-kLog2e, -kLog2e);
    auto zero_row = [](float2 (&v)[NP]) {
#pragma unroll
        for (int p = 0; p < NP; ++p) v[p] = make_float2(0.f, 0.f);
    };
    // dz of the K-1 tokens after a unit (its last dx rows read them): the
    // first rows of the unit walked just before it, kept in carry[k & 1]
    // (rows K-1 .. KW-2 stay zero), or computed for the block's first unit
    float *carry0 = dzs + kProBwdRun * D;
    int st = 0;
#pragma unroll 1
    for (int k = 0; k < n_my; ++k) {
        const int j = j_hi - 1 - k;
        const int b = j / runs, t0 = (j % runs) * kProBwdRun, len = min(kProBwdRun, T - t0);
        float *carry_in = carry0 + (k & 1) * (KW - 1) * D, *carry_out = carry0 + ((k + 1) & 1) * (KW - 1) * D;
        if (threadIdx.x == 0 && k + kProBwdStages - 1 < n_my) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(k + kProBwdStages - 1, st == 0 ? kProBwdStages - 1 : st - 1);
        }
        if (!mbar_wait(&bars[st], (uint32_t)(k / kProBwdStages) & 1u)) {
            record_status(GDR_ERR_TIMEOUT);
            blk_drain<kProBwdStages>(bars, st, k, k, n_my, 1);
            return;
        }
        uint8_t *stage = smem + st * stage_bytes;
        if (t0 == 0 && a.state_in != nullptr && K > 1) {
            constexpr int kPieces = D * (int)sizeof(Tio) / 16;
            for (int i = threadIdx.x; i < (K - 1) * kPieces; i += kBlkThreads) {
                const int r = i / kPieces, q = i % kPieces;
                const Tio *src = static_cast<const Tio *>(a.state_in) + ((size_t)b * (K - 1) + r) * Ctot + col + h * D;
                reinterpret_cast<uint4 *>(stage + (size_t)r * D * sizeof(Tio))[q] =
                    reinterpret_cast<const uint4 *>(src)[q];
            }
            __syncthreads();
        }
        const Tio *sx = reinterpret_cast<const Tio *>(stage) + lane * CPL;
        const Tio *sdy = reinterpret_cast<const Tio *>(stage + xalloc) + lane * CPL;

        // phase 1: dz for tokens t0 .. t0+63 (row r = token t0 + r).  NB
        // consecutive rows per step from a register window of x rows:
        // win[m] = x row r + K - KW + m (stage row r + m' holds the x read by
        // tap m' of row r), so row r + q reads win[q .. q + KW - 1].  dy of
        // row r + q is at dyp + q * dys, its dz goes to dzp + q * D; rows
        // r + nrows .. r + NB - 1 are computed on zeros and dropped.  dy is
        // zero past T (the TMA fill, or the caller), so dz is zero there.
        //   u = SiLU(z) = z sg,  g = dSiLU/dz = sg (1 + z (1 - sg)) = sg + u (1 - sg)
        constexpr int NBW = KW <= 4 ? kProBwdNB : 1, WR = KW + NBW - 1;  // one row per step at K > 4
        auto dz_rows = [&](int r, int nrows, float2(&win)[WR][NP], const Tio *dyp, size_t dys, float *dzp) {
            constexpr int NB = NBW;
            float2 dyv[NB][NP], u[NB][NP], g[NB][NP];
            float ss[NB], ud[NB];
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                if (q < nrows)
                    ld_row<CPL>(dyp + q * dys, reinterpret_cast<float *>(dyv[q]));
                else
                    zero_row(dyv[q]);
                float2 ss2 = make_float2(0.f, 0.f), ud2 = make_float2(0.f, 0.f);
#pragma unroll
                for (int p = 0; p < NP; ++p) {
                    float2 z = bias[p];
#pragma unroll
                    for (int m = 0; m < KW; ++m) z = ffma2(wt[p][m], win[q + m][p], z);
                    const float2 e = fmul2(z, ml2e2);
                    const float2 den = ffma2(make_float2(ex2_ftz(e.x), ex2_ftz(e.y)), one2, one2);
                    const float2 sg = make_float2(rcp_ftz(den.x), rcp_ftz(den.y));
                    u[q][p] = fmul2(z, sg);
                    g[q][p] = ffma2(u[q][p], ffma2(sg, mone2, one2), sg);
                    ss2 = ffma2(u[q][p], u[q][p], ss2);
                    ud2 = ffma2(u[q][p], dyv[q][p], ud2);
                }
                ss[q] = ss2.x + ss2.y;
                ud[q] = ud2.x + ud2.y;
            }
            // L2 reverse: y = u/n, du = (dy - y (y . dy)) / n
            //                        = (dy - u (u . dy) / n^2) / n;
            // both row sums reduce together
            float2 dz[NB][NP];
            if (l2) {
#pragma unroll
                for (int off = 16; off > 0; off >>= 1)
#pragma unroll
                    for (int q = 0; q < NB; ++q) {
                        ss[q] += __shfl_xor_sync(0xffffffffu, ss[q], off);
                        ud[q] += __shfl_xor_sync(0xffffffffu, ud[q], off);
                    }
#pragma unroll
                for (int q = 0; q < NB; ++q) {
                    // zero past T, where u may be all zero (no 0 * inf with eps = 0)
                    const float ninv = t0 + r + q < T ? rsqrt_ftz(ss[q] + a.eps) : 0.f, f = -ud[q] * ninv * ninv;
                    const float2 f2 = make_float2(f, f), n2 = make_float2(ninv, ninv);
#pragma unroll
                    for (int p = 0; p < NP; ++p) dz[q][p] = fmul2(ffma2(u[q][p], f2, dyv[q][p]), fmul2(g[q][p], n2));
                }
            } else {
#pragma unroll
                for (int q = 0; q < NB; ++q)
#pragma unroll
                    for (int p = 0; p < NP; ++p) dz[q][p] = fmul2(dyv[q][p], g[q][p]);
            }
#pragma unroll
            for (int q = 0; q < NB; ++q) {
                if (q >= nrows) break;
                st_row<CPL>(dzp + q * D, reinterpret_cast<const float *>(dz[q]));
                if (r + q < kProBwdRun) {  // the unit's own rows: dw and dbias
#pragma unroll
                    for (int p = 0; p < NP; ++p) {
#pragma unroll
                        for (int m = 0; m < KW; ++m) dwa[p][m] = ffma2(dz[q][p], win[q + m][p], dwa[p][m]);
                        dba[p] = ffma2(dz[q][p], one2, dba[p]);
                    }
                }
                if (r + q < K - 1) {  // the next unit walked (tokens before t0) reads these
                    if (t0 == 0) zero_row(dz[q]);  // ... unless it is another batch's
                    st_row<CPL>(carry_out + (r + q) * D + lane * CPL, reinterpret_cast<const float *>(dz[q]));
                }
            }
        };
        {  // the unit's 64 rows: warp w takes rows 8w .. 8w+7
            const int r0 = warp * kProBwdRowsPerWarp;
            float2 win[WR][NP];
#pragma unroll
            for (int m = 0; m < KW - 1; ++m) {
                const int row = r0 + K - KW + m;
                if (row >= 0)
                    ld_row<CPL>(sx + row * D, reinterpret_cast<float *>(win[m]));
                else
                    zero_row(win[m]);
            }
#pragma unroll
            for (int p = 0; p < kProBwdRowsPerWarp; p += NBW) {
                const int r = r0 + p;
#pragma unroll
                for (int m = KW - 1; m < WR; ++m) ld_row<CPL>(sx + (r + K - KW + m) * D, reinterpret_cast<float *>(win[m]));
                dz_rows(r, NBW, win, sdy + r * D, D, dzs + r * D + lane * CPL);
#pragma unroll
                for (int m = 0; m < KW - 1; ++m)
#pragma unroll
                    for (int c = 0; c < NP; ++c) win[m][c] = win[m + NBW][c];
            }
        }
        if (k == 0 && warp < K - 1) {
            // the block's first unit: dz of token t0 + 64 + warp from global
            // memory (zero past T; the x it reads are tokens t0 + 57 .. t)
            const int r = kProBwdRun + warp, t = t0 + r;
            float2 win[WR][NP];
#pragma unroll
            for (int m = 0; m < WR; ++m) {
                if (t < T && m < KW)
                    ld_row<CPL>(xg + (((size_t)b * T + t + 1 - KW + m) * H) * D + c0, reinterpret_cast<float *>(win[m]));
                else
                    zero_row(win[m]);
            }
            dz_rows(r, t < T ? 1 : 0, win, dyg + (((size_t)b * T + t) * H) * D + c0, 0, carry_in + warp * D + lane * CPL);
            if (t >= T) {
                float2 zero[NP];
                zero_row(zero);
                st_row<CPL>(carry_in + warp * D + lane * CPL, reinterpret_cast<const float *>(zero));
            }
        }
        __syncthreads();

        // phase 2: dx[i] = sum_j w[j] dz[i + K-1-j], from a window of dz rows
        // dzw[n] = dz row i + n (n < KW), which tap K-1-n = wt[.][KW-1-n]
        // multiplies (zero for n >= K); rows 64 .. 64+KW-2 are carry_in's
        auto dx_row = [&](int i, const float2 (&dzw)[KW][NP]) {
            if (i >= len) return;  // past the end of a ragged last unit
            float2 acc[NP];
#pragma unroll
            for (int p = 0; p < NP; ++p) {
                float2 v = make_float2(0.f, 0.f);
#pragma unroll
                for (int n = 0; n < KW; ++n) v = ffma2(wt[p][KW - 1 - n], dzw[n][p], v);
                acc[p] = v;
            }
            const int ms = t0 + i - (T - (K - 1));  // slot of this x in the returned state
            if (dso != nullptr && ms >= 0) {
                float2 gs[NP];
                ld_row<CPL>(dso + ((size_t)b * (K - 1) + ms) * Ctot + col + c0, reinterpret_cast<float *>(gs));
#pragma unroll
                for (int p = 0; p < NP; ++p) acc[p] = ffma2(gs[p], one2, acc[p]);
            }
            if (i >= 0) {
                st_row<CPL>(dxb + ((size_t)b * T + t0 + i) * H * D + c0, reinterpret_cast<const float *>(acc));
            } else {
                st_row<CPL>(dsi + ((size_t)b * (K - 1) + (K - 1 + i)) * Ctot + col + c0,
                            reinterpret_cast<const float *>(acc));
            }
        };
        auto dz_row_ptr = [&](int row) {
            return (row < kProBwdRun ? dzs + row * D : carry_in + (row - kProBwdRun) * D) + lane * CPL;
        };
        {
            const int i0 = warp * kProBwdRowsPerWarp;
            float2 dzw[KW][NP];
#pragma unroll
            for (int n = 0; n < KW - 1; ++n) ld_row<CPL>(dz_row_ptr(i0 + n), reinterpret_cast<float *>(dzw[n]));
#pragma unroll
            for (int p = 0; p < kProBwdRowsPerWarp; ++p) {
                ld_row<CPL>(dz_row_ptr(i0 + p + KW - 1), reinterpret_cast<float *>(dzw[KW - 1]));
                dx_row(i0 + p, dzw);
#pragma unroll
                for (int n = 0; n < KW - 1; ++n)
#pragma unroll
                    for (int c = 0; c < NP; ++c) dzw[n][c] = dzw[n + 1][c];
            }
        }
        if (t0 == 0 && dsi != nullptr && warp < K - 1) {  // the carried-in state's rows
            const int i = warp - (K - 1);
            float2 dzw[KW][NP];
#pragma unroll
            for (int n = 0; n < KW; ++n) {
                if (i + n >= 0)
                    ld_row<CPL>(dz_row_ptr(i + n), reinterpret_cast<float *>(dzw[n]));
                else
                    zero_row(dzw[n]);
            }
            dx_row(i, dzw);
        }
        __syncthreads();
        st = st == kProBwdStages - 1 ? 0 : st + 1;
    }
    // every issued copy has been waited on: stage memory holds the warp sums
    float *red = reinterpret_cast<float *>(smem);
    constexpr int E = D * (KW + 1);
#pragma unroll
    for (int p = 0; p < NP; ++p) {
        float *row0 = red + warp * E + (lane * CPL + 2 * p) * (KW + 1), *row1 = row0 + (KW + 1);
#pragma unroll
        for (int m = 0; m < KW; ++m)
            if (m >= KW - K) {
                row0[m - (KW - K)] = dwa[p][m].x;
                row1[m - (KW - K)] = dwa[p][m].y;
            }
        row0[KW] = dba[p].x;
        row1[KW] = dba[p].y;
    }
    __syncthreads();
    float *out = a.partial + (size_t)blockIdx.x * a.partial_stride;
    for (int e = threadIdx.x; e < E; e += kBlkThreads) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < NW; ++w) acc += red[w * E + e];
        out[e] = acc;
    }
}

template <typename Tio, int DQK, int DV, int KW>
__global__ void __launch_bounds__(kBlkThreads)
    gdr_prologue_bwd_kernel(const PrologueBwdArgs a, int stage_bytes, int xalloc,
                            const __grid_constant__ CUtensorMap tm_xq, const __grid_constant__ CUtensorMap tm_xk,
                            const __grid_constant__ CUtensorMap tm_xv, const __grid_constant__ CUtensorMap tm_dq,
                            const __grid_constant__ CUtensorMap tm_dk, const __grid_constant__ CUtensorMap tm_dv) {
    using namespace sm100;
    constexpr int DMAX = DQK > DV ? DQK : DV;
    extern __shared__ __align__(128) uint8_t blk_smem[];
    uint8_t *smem = blk_smem;
    float *dzs = reinterpret_cast<float *>(smem + kProBwdStages * stage_bytes);
    uint64_t *bars = reinterpret_cast<uint64_t *>(dzs + (kProBwdRun + 2 * (KW - 1)) * DMAX);
    const int P = 3 * a.H, pair = blockIdx.x % P, idx = blockIdx.x / P, G = gridDim.x / P;
    const int s = pair / a.H, h = pair % a.H;
    if (threadIdx.x == 0) {
        for (int i = 0; i < kProBwdStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
    }
    // the carried dz rows past K-2 are read (by taps that are zero) and never written
    for (int i = threadIdx.x; i < (kProBwdRun + 2 * (KW - 1)) * DMAX; i += kBlkThreads) dzs[i] = 0.f;
    __syncthreads();
    if (s == 0)
        prologue_bwd_block<Tio, DQK, KW>(a, &tm_xq, &tm_dq, s, h, idx, G, smem, stage_bytes, xalloc, dzs, bars);
    else if (s == 1)
        prologue_bwd_block<Tio, DQK, KW>(a, &tm_xk, &tm_dk, s, h, idx, G, smem, stage_bytes, xalloc, dzs, bars);
    else
        prologue_bwd_block<Tio, DV, KW>(a, &tm_xv, &tm_dv, s, h, idx, G, smem, stage_bytes, xalloc, dzs, bars);
}

// dw[s][(h*D + c)*K + j] and dbias[s][h*D + c]: the sums over the G blocks of
// pair (s, h) in block order.  One block per pair.
struct PrologueBwdSum {
    int H, dk, dv, K, KW, G, stride;
    const float *partial;
    float *dw[3];
    float *dbias[3];  // each may be null (not written)
};

__global__ void prologue_bwd_sum_kernel(const PrologueBwdSum p) {
    const int P = 3 * p.H, pair = blockIdx.x, s = pair / p.H, h = pair % p.H;
    const int D = s < 2 ? p.dk : p.dv;
    float *dw = s == 0 ? p.dw[0] : s == 1 ? p.dw[1] : p.dw[2];
    float *db = s == 0 ? p.dbias[0] : s == 1 ? p.dbias[1] : p.dbias[2];
    for (int e = threadIdx.x; e < D * (p.K + 1); e += blockDim.x) {
        const int c = e / (p.K + 1), m = e % (p.K + 1);
        const int slot = c * (p.KW + 1) + (m < p.K ? m : p.KW);
        float acc = 0.f;
        for (int g = 0; g < p.G; ++g) acc += p.partial[(size_t)(g * P + pair) * p.stride + slot];
        if (m < p.K)
            dw[(size_t)(h * D + c) * p.K + m] = acc;
        else if (db != nullptr)
            db[h * D + c] = acc;
    }
}

// ---- epilogue ---------------------------------------------------------------------
// y = o / sqrt(mean(o^2) + eps) * weight * SiLU(g) per row of dv channels;
// g == nullptr leaves out the gate.  Rows are the B*T*H (token, head) pairs,
// contiguous in memory, so a unit of 64 rows of o (and of g) arrives by one
// bulk copy each; a ring of kBlkStages units per block keeps copies in flight
// while warps compute (warp w: rows kRowsPerWarp*w .. kRowsPerWarp*(w+1)-1 of the unit, four rows at 512 threads).
constexpr int kEpilogueRows = 64;
constexpr int kEpiThreads = 512;  // 16 warps: 4 rows of a unit each

template <typename Tio, int CPL>
__global__ void __launch_bounds__(kEpiThreads)
    gdr_epilogue_kernel(long long rows, const Tio *__restrict__ o, const Tio *__restrict__ g,
                        const float *__restrict__ weight, float eps, Tio *__restrict__ y) {
    using namespace sm100;
    constexpr int D = CPL * 32;
    constexpr int kTile = kEpilogueRows * D * (int)sizeof(Tio);  // one tensor's unit
    constexpr int kRowsPerWarp = kEpilogueRows / (kEpiThreads / 32);
    extern __shared__ __align__(128) uint8_t blk_smem[];
    uint8_t *smem = blk_smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + kBlkStages * 2 * kTile);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long units = (rows + kEpilogueRows - 1) / kEpilogueRows;
    auto issue = [&](long long uu, int sidx) {  // one thread
        const long long r0 = uu * kEpilogueRows;
        const uint32_t bytes = (uint32_t)min((long long)kEpilogueRows, rows - r0) * D * (uint32_t)sizeof(Tio);
        mbar_expect_tx(&bars[sidx], g ? 2 * bytes : bytes);
        bulk_load_g2s(smem + sidx * 2 * kTile, o + r0 * D, bytes, &bars[sidx]);
        if (g) bulk_load_g2s(smem + sidx * 2 * kTile + kTile, g + r0 * D, bytes, &bars[sidx]);
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < kBlkStages; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        for (int k = 0; k < kBlkStages - 1; ++k)
            if (blockIdx.x + (long long)k * gridDim.x < units) issue(blockIdx.x + (long long)k * gridDim.x, k);
    }
    __syncthreads();
    float wl[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) wl[c] = __ldg(weight + lane * CPL + c);
    int st = 0;
#pragma unroll 1
    for (int k = 0;; ++k) {
        const long long u = blockIdx.x + (long long)k * gridDim.x;
        if (u >= units) break;
        const long long un = u + (long long)(kBlkStages - 1) * gridDim.x;
        if (threadIdx.x == 0 && un < units) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(un, st == 0 ? kBlkStages - 1 : st - 1);
        }
        if (!mbar_wait(&bars[st], (uint32_t)(k / kBlkStages) & 1u)) {
            record_status(GDR_ERR_TIMEOUT);
            blk_drain<kBlkStages>(bars, st, k, u, units, gridDim.x);
            return;
        }
        const Tio *so = reinterpret_cast<const Tio *>(smem + st * 2 * kTile) + lane * CPL;
        const Tio *sg = so + kTile / sizeof(Tio);
        const long long r0 = u * kEpilogueRows;
        const int n = (int)min((long long)kEpilogueRows, rows - r0);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int i = warp * kRowsPerWarp + r;
            if (i >= n) break;
            float ov[CPL], gv[CPL], ss = 0.f;
            ld_row<CPL>(so + i * D, ov);
            if (g) ld_row<CPL>(sg + i * D, gv);
#pragma unroll
            for (int c = 0; c < CPL; ++c) ss = fmaf(ov[c], ov[c], ss);
            const float inv = rsqrt_ftz(warp_sum(ss, 32) * (1.f / D) + eps);
            float out[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) out[c] = ov[c] * inv * wl[c] * (g ? silu_f(gv[c]) : 1.f);
            st_row<CPL>(y + (size_t)(r0 + i) * D + lane * CPL, out);
        }
        __syncthreads();
        st = st == kBlkStages - 1 ? 0 : st + 1;
    }
}

// ---- epilogue backward ------------------------------------------------------------
// Reverse mode of y = a * weight * s, a = o * r, r = 1/sqrt(mean(o^2) + eps),
// s = SiLU(g) (s = 1 without a gate), for an incoming dy:
//   dg      = dy a weight sig (1 + g (1 - sig)),   sig = 1/(1 + e^-g)
//   da      = dy weight s
//   do      = r (da - a mean(da a))
//   dweight = sum over rows of dy a s.
// Same unit walk as the forward (64 rows, one bulk copy per tensor: o, g, dy),
// NS stages deep.  Each lane keeps its channels' dweight partial sums over its
// rows in registers; at the end the block sums its 16 warps in warp order and
// writes one row of `partial` [gridDim.x, D], which a second launch sums over
// blocks in block order -- the result is independent of timing.
constexpr int kEpiBwdMaxBlocks = 1024;  // partial rows: the workspace bound

template <typename Tio, int CPL, int NS>
__global__ void __launch_bounds__(kEpiThreads)
    gdr_epilogue_bwd_kernel(long long rows, const Tio *__restrict__ o, const Tio *__restrict__ g,
                            const Tio *__restrict__ dy, const float *__restrict__ weight, float eps,
                            Tio *__restrict__ dO, Tio *__restrict__ dg, float *__restrict__ partial) {
    using namespace sm100;
    constexpr int D = CPL * 32;
    constexpr int kTile = kEpilogueRows * D * (int)sizeof(Tio);
    constexpr int kWarps = kEpiThreads / 32;
    constexpr int kRowsPerWarp = kEpilogueRows / kWarps;
    extern __shared__ __align__(128) uint8_t blk_smem[];
    uint8_t *smem = blk_smem;
    uint64_t *bars = reinterpret_cast<uint64_t *>(smem + NS * 3 * kTile);
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const long long units = (rows + kEpilogueRows - 1) / kEpilogueRows;
    auto issue = [&](long long uu, int sidx) {  // one thread
        const long long r0 = uu * kEpilogueRows;
        const uint32_t bytes = (uint32_t)min((long long)kEpilogueRows, rows - r0) * D * (uint32_t)sizeof(Tio);
        uint8_t *dst = smem + sidx * 3 * kTile;
        mbar_expect_tx(&bars[sidx], g ? 3 * bytes : 2 * bytes);
        bulk_load_g2s(dst, o + r0 * D, bytes, &bars[sidx]);
        bulk_load_g2s(dst + 2 * kTile, dy + r0 * D, bytes, &bars[sidx]);
        if (g) bulk_load_g2s(dst + kTile, g + r0 * D, bytes, &bars[sidx]);
    };
    if (threadIdx.x == 0) {
        for (int i = 0; i < NS; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        for (int k = 0; k < NS - 1; ++k)
            if (blockIdx.x + (long long)k * gridDim.x < units) issue(blockIdx.x + (long long)k * gridDim.x, k);
    }
    __syncthreads();
    float wl[CPL], dwp[CPL];
#pragma unroll
    for (int c = 0; c < CPL; ++c) {
        wl[c] = __ldg(weight + lane * CPL + c);
        dwp[c] = 0.f;
    }
    int st = 0;
#pragma unroll 1
    for (int k = 0;; ++k) {
        const long long u = blockIdx.x + (long long)k * gridDim.x;
        if (u >= units) break;
        const long long un = u + (long long)(NS - 1) * gridDim.x;
        if (threadIdx.x == 0 && un < units) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(un, st == 0 ? NS - 1 : st - 1);
        }
        if (!mbar_wait(&bars[st], (uint32_t)(k / NS) & 1u)) {
            record_status(GDR_ERR_TIMEOUT);
            blk_drain<NS>(bars, st, k, u, units, gridDim.x);
            return;
        }
        const Tio *so = reinterpret_cast<const Tio *>(smem + st * 3 * kTile) + lane * CPL;
        const Tio *sg = so + kTile / sizeof(Tio);
        const Tio *sd = so + 2 * (kTile / sizeof(Tio));
        const long long r0 = u * kEpilogueRows;
        const int n = (int)min((long long)kEpilogueRows, rows - r0);
#pragma unroll
        for (int r = 0; r < kRowsPerWarp; ++r) {
            const int i = warp * kRowsPerWarp + r;
            if (i >= n) break;
            float ov[CPL], gv[CPL], dv_[CPL], ss = 0.f;
            ld_row<CPL>(so + i * D, ov);
            ld_row<CPL>(sd + i * D, dv_);
            if (g) ld_row<CPL>(sg + i * D, gv);
#pragma unroll
            for (int c = 0; c < CPL; ++c) ss = fmaf(ov[c], ov[c], ss);
            const float inv = rsqrt_ftz(warp_sum(ss, 32) * (1.f / D) + eps);
            float a[CPL], da[CPL], dgo[CPL], dot = 0.f;
#pragma unroll
            for (int c = 0; c < CPL; ++c) {
                a[c] = ov[c] * inv;
                float s = 1.f;
                if (g) {
                    const float z = gv[c];
                    const float sig = rcp_ftz(1.f + ex2_ftz(-kLog2e * z));
                    s = z * sig;
                    dgo[c] = dv_[c] * a[c] * wl[c] * sig * fmaf(z, 1.f - sig, 1.f);
                }
                const float dys = dv_[c] * s;
                da[c] = dys * wl[c];
                dwp[c] = fmaf(dys, a[c], dwp[c]);
                dot = fmaf(da[c], a[c], dot);
            }
            dot = warp_sum(dot, 32) * (1.f / D);
            float out[CPL];
#pragma unroll
            for (int c = 0; c < CPL; ++c) out[c] = inv * fmaf(-a[c], dot, da[c]);
            const size_t off = (size_t)(r0 + i) * D + lane * CPL;
            st_row<CPL>(dO + off, out);
            if (g) st_row<CPL>(dg + off, dgo);
        }
        __syncthreads();
        st = st == NS - 1 ? 0 : st + 1;
    }
    // every issued copy has been waited on: the stages are free for the sums
    float *red = reinterpret_cast<float *>(smem);
#pragma unroll
    for (int c = 0; c < CPL; ++c) red[warp * D + lane * CPL + c] = dwp[c];
    __syncthreads();
    if (threadIdx.x < D) {
        float acc = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) acc += red[w * D + threadIdx.x];
        partial[(size_t)blockIdx.x * D + threadIdx.x] = acc;
    }
}

// dweight[c] = sum over b < nblk of partial[b, c], in block order.
__global__ void epilogue_dweight_sum_kernel(int nblk, int D, const float *__restrict__ partial,
                                            float *__restrict__ dweight) {
    const int c = threadIdx.x;
    if (c >= D) return;
    float acc = 0.f;
    for (int b = 0; b < nblk; ++b) acc += partial[(size_t)b * D + c];
    dweight[c] = acc;
}

// Grid = SMs x resident blocks of the kernel (capped by the work), so the
// stride loop covers the units in whole waves.
// (Queried on every launch: the occupancy call is a cheap host query, and a
// cache keyed on the kernel's type would mix instantiations whose shared
// memory differs.)
template <typename Kern>
inline int resident_grid(Kern kernel, long long warps_needed, int smem = 0, int threads = kBlkThreads) {
    int dev = 0, nb = 0, sms = 0;
    if (cudaGetDevice(&dev) != cudaSuccess ||
        cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess ||
        cudaOccupancyMaxActiveBlocksPerMultiprocessor(&nb, kernel, threads, smem) != cudaSuccess)
        return 0;
    const int per_sm = nb > 0 ? nb : 1;
    const long long blocks = (warps_needed + threads / 32 - 1) / (threads / 32);
    return (int)std::min<long long>(blocks, (long long)sms * per_sm);
}

// 4-D map over one projected stream [B, T, H, d]: box = d channels x 1 head x
// `rows` tokens x 1 batch, no swizzle (the stage is row-major [rows][d]);
// coordinates outside the tensor read as zero.
template <typename Tio>
inline bool make_prologue_map(CUtensorMap *map, const void *base, int B, int T, int H, int d, int rows) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t es = sizeof(Tio);
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * es, (cuuint64_t)H * d * es, (cuuint64_t)T * H * d * es};
    const cuuint32_t box[4] = {(cuuint32_t)d, 1, (cuuint32_t)rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    const CUtensorMapDataType dt = sizeof(Tio) == 4 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    return enc(map, dt, 4, const_cast<void *>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <typename Tio, int DQK, int DV>
inline cudaError_t launch_prologue_t(const PrologueArgs &a, cudaStream_t stream) {
    auto kern = a.K <= 4 ? gdr_prologue_kernel<Tio, DQK, DV, 4> : gdr_prologue_kernel<Tio, DQK, DV, kConvMax>;
    constexpr int DMAX = DQK > DV ? DQK : DV;
    const int stage_bytes = kPrologueRows * DMAX * (int)sizeof(Tio);
    const int smem = kProStages * (stage_bytes + 8);
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    CUtensorMap mq, mk, mv;
    if (!make_prologue_map<Tio>(&mq, a.x[0], a.B, a.T, a.H, a.dk, kPrologueRun + a.K - 1) ||
        !make_prologue_map<Tio>(&mk, a.x[1], a.B, a.T, a.H, a.dk, kPrologueRun + a.K - 1) ||
        !make_prologue_map<Tio>(&mv, a.x[2], a.B, a.T, a.H, a.dv, kPrologueRun + a.K - 1))
        return cudaErrorInvalidValue;
    // 3H (stream, head) pairs x G blocks each, G filling the resident slots
    const long long pairs = 3LL * a.H, units = (long long)a.B * ((a.T + kPrologueRun - 1) / kPrologueRun);
    const long long slots = resident_grid(kern, 1LL << 40, smem);
    if (slots <= 0) return cudaErrorInvalidConfiguration;
    const long long G = std::max(1LL, std::min(units, slots / pairs));
    if (pairs * G >= (1LL << 31)) return cudaErrorInvalidConfiguration;
    kern<<<(unsigned)(pairs * G), kBlkThreads, smem, stream>>>(a, stage_bytes, mq, mk, mv);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

template <typename Tio>
inline cudaError_t launch_prologue(const PrologueArgs &a, cudaStream_t stream) {
    if (a.dk == 128 && a.dv == 128) return launch_prologue_t<Tio, 128, 128>(a, stream);
    if (a.dk == 128 && a.dv == 64) return launch_prologue_t<Tio, 128, 64>(a, stream);
    if (a.dk == 64 && a.dv == 128) return launch_prologue_t<Tio, 64, 128>(a, stream);
    return launch_prologue_t<Tio, 64, 64>(a, stream);
}

template <typename Tio>
inline cudaError_t launch_epilogue(long long rows, int dv, const void *o, const void *g, const float *weight,
                                   float eps, void *y, cudaStream_t stream) {
    auto run = [&](auto kern, int d) -> cudaError_t {
        const int smem = kBlkStages * 2 * kEpilogueRows * d * (int)sizeof(Tio) + 8 * kBlkStages;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const long long units = (rows + kEpilogueRows - 1) / kEpilogueRows;
        const int grid = resident_grid(kern, units * (kEpiThreads / 32), smem, kEpiThreads);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        kern<<<grid, kEpiThreads, smem, stream>>>(rows, static_cast<const Tio *>(o), static_cast<const Tio *>(g),
                                                  weight, eps, static_cast<Tio *>(y));
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cudaGetLastError();
    };
    return dv == 128 ? run(gdr_epilogue_kernel<Tio, 4>, 128) : run(gdr_epilogue_kernel<Tio, 2>, 64);
}

template <typename Tio>
inline cudaError_t launch_epilogue_bwd(long long rows, int dv, const void *o, const void *g, const void *dy,
                                       const float *weight, float eps, void *dO, void *dg, float *dweight,
                                       float *partial, cudaStream_t stream) {
    // 3 tensors x 2 stages x 64 rows: 96 KB for bf16, so two blocks (32 warps)
    // share an SM; a third stage at one block per SM measured 12 % slower.
    constexpr int NS = 2;
    auto run = [&](auto kern, int d) -> cudaError_t {
        const int smem = NS * 3 * kEpilogueRows * d * (int)sizeof(Tio) + 8 * NS;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        const long long units = (rows + kEpilogueRows - 1) / kEpilogueRows;
        const int grid = std::min(resident_grid(kern, units * (kEpiThreads / 32), smem, kEpiThreads), kEpiBwdMaxBlocks);
        if (grid <= 0) return cudaErrorInvalidConfiguration;
        kern<<<grid, kEpiThreads, smem, stream>>>(rows, static_cast<const Tio *>(o), static_cast<const Tio *>(g),
                                                  static_cast<const Tio *>(dy), weight, eps, static_cast<Tio *>(dO),
                                                  static_cast<Tio *>(dg), partial);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        epilogue_dweight_sum_kernel<<<1, d, 0, stream>>>(grid, d, partial, dweight);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cudaGetLastError();
    };
    return dv == 128 ? run(gdr_epilogue_bwd_kernel<Tio, 4, NS>, 128) : run(gdr_epilogue_bwd_kernel<Tio, 2, NS>, 64);
}

// Grid: 3H pairs x G blocks, G filling the resident slots (at most
// kProBwdMaxG); then one block per pair for the fixed-order sums.
template <typename Tio, int DQK, int DV, int KW>
inline cudaError_t launch_prologue_bwd_kw(PrologueBwdArgs a, float *const dw[3], float *const dbias[3],
                                          cudaStream_t stream) {
    constexpr int DMAX = DQK > DV ? DQK : DV;
    auto kern = gdr_prologue_bwd_kernel<Tio, DQK, DV, KW>;
    const int xalloc = (kProBwdRun + KW - 1) * DMAX * (int)sizeof(Tio);
    const int stage_bytes = xalloc + kProBwdRun * DMAX * (int)sizeof(Tio);
    static_assert((kBlkThreads / 32) * DMAX * (KW + 1) * 4 <= kProBwdStages * (2 * kProBwdRun + KW - 1) * DMAX * 2,
                  "warp sums must fit in the stages");
    const int smem = kProBwdStages * stage_bytes + (kProBwdRun + 2 * (KW - 1)) * DMAX * 4 + 8 * kProBwdStages;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    const int K = a.K;
    CUtensorMap mx[3], mdy[3];
    for (int s = 0; s < 3; ++s) {
        const int d = s < 2 ? a.dk : a.dv;
        if (!make_prologue_map<Tio>(&mx[s], a.x[s], a.B, a.T, a.H, d, kProBwdRun + K - 1) ||
            !make_prologue_map<Tio>(&mdy[s], a.dy[s], a.B, a.T, a.H, d, kProBwdRun))
            return cudaErrorInvalidValue;
    }
    const long long pairs = 3LL * a.H, units = (long long)a.B * ((a.T + kProBwdRun - 1) / kProBwdRun);
    const long long slots = resident_grid(kern, 1LL << 40, smem);
    if (slots <= 0) return cudaErrorInvalidConfiguration;
    const long long G = std::max(1LL, std::min({units, slots / pairs, (long long)kProBwdMaxG}));
    if (pairs * G >= (1LL << 31)) return cudaErrorInvalidConfiguration;
    a.partial_stride = DMAX * (KW + 1);
    kern<<<(unsigned)(pairs * G), kBlkThreads, smem, stream>>>(a, stage_bytes, xalloc, mx[0], mx[1], mx[2], mdy[0],
                                                              mdy[1], mdy[2]);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    PrologueBwdSum p{};
    p.H = a.H; p.dk = a.dk; p.dv = a.dv; p.K = K; p.KW = KW; p.G = (int)G; p.stride = a.partial_stride;
    p.partial = a.partial;
    for (int s = 0; s < 3; ++s) {
        p.dw[s] = dw[s];
        p.dbias[s] = dbias[s];
    }
    prologue_bwd_sum_kernel<<<(unsigned)pairs, kBlkThreads, 0, stream>>>(p);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

// Workspace of the per-block partial sums.
inline size_t prologue_bwd_workspace(int H, int dk, int dv, int K) {
    const int KW = K <= 4 ? 4 : kConvMax;
    return (size_t)3 * H * kProBwdMaxG * std::max(dk, dv) * (KW + 1) * sizeof(float);
}

template <typename Tio, int DQK, int DV>
inline cudaError_t launch_prologue_bwd_t(const PrologueBwdArgs &a, float *const dw[3], float *const dbias[3],
                                         cudaStream_t stream) {
    return a.K <= 4 ? launch_prologue_bwd_kw<Tio, DQK, DV, 4>(a, dw, dbias, stream)
                    : launch_prologue_bwd_kw<Tio, DQK, DV, kConvMax>(a, dw, dbias, stream);
}

template <typename Tio>
inline cudaError_t launch_prologue_bwd(const PrologueBwdArgs &a, float *const dw[3], float *const dbias[3],
                                       cudaStream_t stream) {
    if (a.dk == 128 && a.dv == 128) return launch_prologue_bwd_t<Tio, 128, 128>(a, dw, dbias, stream);
    if (a.dk == 128 && a.dv == 64) return launch_prologue_bwd_t<Tio, 128, 64>(a, dw, dbias, stream);
    if (a.dk == 64 && a.dv == 128) return launch_prologue_bwd_t<Tio, 64, 128>(a, dw, dbias, stream);
    return launch_prologue_bwd_t<Tio, 64, 64>(a, dw, dbias, stream);
}

}  // namespace gdr
