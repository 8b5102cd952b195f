// bwd2_tc.cuh -- the chunk products and the per-element chain rule of the
// Gated DeltaNet-2 backward on tcgen05, one CTA per (b, h, chunk) (bf16 with
// dk = 128).
//
// In the chunk form of the backward (bwd2_simt.cuh header; Gated DeltaNet-2,
// agihunt.info/papers/2605.22791, the Gated Delta Rule-2 paragraph, with the
// chain rule through the gates inside the dot products) the gradients of the
// chunk operands are
//     dKBE = -dR S + dA KiE,  dQE = dO S + dP KiE,
//     dKiE = dA^T KBE + dP^T QE + (U D) Diag(E_C),
// with KBE = K*B*E, QE = Q*E, KiE = K/E.  The terms in S and D belong to the
// value rows, so the reverse pass over slices of value rows writes them as
// per-slice partials; dA and dP are sums over value rows too, so each slice
// writes its dA and dP and this kernel adds the slices first and then forms
// the C x C x dk products once per chunk-head, on the tensor cores with the
// key channel on M = 128:
//     [dKBE^T | dQE^T] = KiE^T [dA ; dP]^T      (N = 128, K = C)
//     dKiE^T = KBE^T dA + QE^T dP               (N = 64,  K = C, two groups)
// (bf16 operands, fp32 accumulation in TMEM).  Thread j then owns key channel
// j: it adds the slices' partials, applies dK = dKBE B E + dKiE / E,
// dB = dKBE K E, dQ = dQE E, and forms dlog alpha as the in-chunk suffix sum
// of dG = dKBE KBE + dQE QE - dKiE KiE (plus E_C dE_C on the last token).
// A chunk that the reverse pass walked token by token (a channel decaying
// past e^80) holds per-token partials instead and is summed without E; a
// chunk decaying past e^20 (where the bf16 operands K/E and K*B*E would span
// more than that range) had all its products formed in fp32 by the reverse
// pass and is only summed here.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdr {

// How a chunk is differentiated, from its largest per-channel decay span
// -G_C: up to kBwd2TcSpan the products with dA and dP run on the tensor cores
// (bf16 operands K/E, K*B*E, Q*E span e^span there), up to 80 in fp32 in the
// reverse pass, beyond that token by token.
constexpr float kBwd2TcSpan = 20.f;
enum : int { kChunkTc = 0, kChunkExact = 1, kChunkF32 = 2 };

constexpr int kBwd2TcThreads = 512;

struct Bwd2TcSmem {
    static constexpr uint32_t oKI = 0;          // K/E  [r][j]: two 64-channel halves, 8 KB each
    static constexpr uint32_t oKB = 16384;      // K*B*E
    static constexpr uint32_t oQE = 32768;      // Q*E
    static constexpr uint32_t oAP = 49152;      // [dA ; dP]: 128 rows x 64 columns, 16 KB
    static constexpr uint32_t oScan = 65536;    // [4][128] fp32: per-quarter totals of the scans
    static constexpr uint32_t oBar = oScan + 2048;
    static constexpr uint32_t kBytes = oBar + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;
};

// NS: slices of value rows (dv / 32), a compile-time constant so that the
// slices' partial loads of a token are issued together.  Thread (warp w,
// lane l) owns key channel j = 32 (w % 4) + l -- TMEM lane j -- and the 16
// tokens r = 16 (w / 4) .. of the chunk, which are its accumulator columns;
// the prefix sum of the gates and the suffix sum of dG run as two-phase scans
// over the four token quarters.
// The chunk ch of (b*H + h) = bh.
template <typename Tio, int NS>
__device__ __forceinline__ void gdr2_bwd_chunk_tc_body(
    int T, int H, const Tio *__restrict__ q, const Tio *__restrict__ k, const float *__restrict__ log_alpha,
    const float *__restrict__ bgate, const float *__restrict__ part_kb, const float *__restrict__ part_qe,
    const float *__restrict__ part_ki, const float *__restrict__ part_ec, const float *__restrict__ part_x,
    const int *__restrict__ exact_flags, const float *__restrict__ dAP, Tio *__restrict__ dq, Tio *__restrict__ dk,
    float *__restrict__ dlog_alpha, float *__restrict__ db, size_t BTH, int bh, int ch) {
    using L = Bwd2TcSmem;
    using namespace sm100;
    constexpr int DK = 128, RQ = kChunk / 4;  // tokens per quarter
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int nchunks = (T + kChunk - 1) / kChunk;
    const int b = bh / H, h = bh % H;
    const int c0 = ch * kChunk, n = min(kChunk, T - c0);
    const size_t tok0 = ((size_t)b * T + c0) * H + h;
    const size_t nbh = BTH / T;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int j = (warp & 3) * 32 + lane, rq = warp >> 2, r0 = rq * RQ;
    const int mode = exact_flags[(size_t)bh * nchunks + ch];

    if (mode == 1) {
        // token-by-token partials: S_t^T do (part_qe), X = P^T gk (part_ki),
        // G^T e (part_kb), sum_i P_ij G_ij (part_x)
#pragma unroll 4
        for (int r = r0; r < r0 + RQ; ++r) {
            if (r >= n) break;
            const size_t off = (tok0 + (size_t)r * H) * DK + j;
            float pq = 0.f, x = 0.f, y = 0.f, z = 0.f;
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                pq += part_qe[(size_t)s * BTH * DK + off];
                x += part_ki[(size_t)s * BTH * DK + off];
                y += part_kb[(size_t)s * BTH * DK + off];
                z += part_x[(size_t)s * BTH * DK + off];
            }
            const float kv = to_f32(k[off]), bv = bgate[off];
            dq[off] = from_f32<Tio>(pq);
            dk[off] = from_f32<Tio>(fmaf(-bv, x, y));
            db[off] = -kv * x;
            dlog_alpha[off] = fmaf(-bv * kv, x, z);
        }
        return;
    }
    const bool use_mma = mode == 0;  // 2: the reverse pass formed the products in fp32 (strong decay)
    uint64_t *bar = reinterpret_cast<uint64_t *>(sm + L::oBar);
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar + 1);
    float *scan = reinterpret_cast<float *>(sm + L::oScan);  // [4][DK]
    if (tid == 0) {
        mbar_init(bar, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 256);

    // G (per-channel cumulative log decay): this quarter's sums, then the
    // earlier quarters' totals; rows past T are identity tokens (zeros)
    float gl = 0.f;
#pragma unroll
    for (int i = 0; i < RQ; ++i) {
        const int r = r0 + i;
        gl += r < n ? log_alpha[(tok0 + (size_t)r * H) * DK + j] : 0.f;
    }
    scan[rq * DK + j] = gl;
    __syncthreads();
    float g0 = 0.f, gC = 0.f;  // G before this quarter; G of the whole chunk
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const float t = scan[u * DK + j];
        if (u < rq) g0 += t;
        gC += t;
    }
    {   // the bf16 operand tiles, channel j of this quarter's rows
        const int half = j >> 6, jj = j & 63;
        float g = g0;
#pragma unroll
        for (int i = 0; i < RQ; ++i) {
            const int r = r0 + i;
            const bool ok = r < n;
            const size_t off = (tok0 + (size_t)r * H) * DK + j;
            g += ok ? log_alpha[off] : 0.f;
            const float e = expf(g);
            const float kv = ok ? to_f32(k[off]) : 0.f, qv = ok ? to_f32(q[off]) : 0.f, bv = ok ? bgate[off] : 0.f;
            const uint32_t po = half * 8192 + sw128_offset(r, jj >> 3) + (jj & 7) * 2;
            *reinterpret_cast<__nv_bfloat16 *>(sm + L::oKI + po) = __float2bfloat16_rn(kv / e);
            *reinterpret_cast<__nv_bfloat16 *>(sm + L::oKB + po) = __float2bfloat16_rn(kv * bv * e);
            *reinterpret_cast<__nv_bfloat16 *>(sm + L::oQE + po) = __float2bfloat16_rn(qv * e);
        }
    }
    // dA and dP of this chunk: the sum over slices of value rows, as bf16 [r][i]
    if (use_mma) {
        const size_t stride = (size_t)nbh * nchunks * 2 * kChunk * kChunk;  // one slice
        const float *src = dAP + ((size_t)bh * nchunks + ch) * 2 * kChunk * kChunk;
#pragma unroll 2
        for (int it = 0; it < 2 * kChunk * kChunk / (4 * kBwd2TcThreads); ++it) {
            const int idx = (it * kBwd2TcThreads + tid) * 4;
            float4 acc = *reinterpret_cast<const float4 *>(src + idx);
#pragma unroll
            for (int s = 1; s < NS; ++s) {
                const float4 x = *reinterpret_cast<const float4 *>(src + (size_t)s * stride + idx);
                acc.x += x.x; acc.y += x.y; acc.z += x.z; acc.w += x.w;
            }
            const int row = idx / kChunk, col = idx % kChunk;  // row 0-63 dA, 64-127 dP
            st_sw_bf16x2(sm + L::oAP, row, col, acc.x, acc.y);
            st_sw_bf16x2(sm + L::oAP, row, col + 2, acc.z, acc.w);
        }
    }
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = *tmem_slot;
    int fail = 0;
    if (tid == 0 && use_mma) {
        const uint32_t sbase = smem_u32(sm);
        const uint32_t ki = sbase + L::oKI, kb = sbase + L::oKB, qe = sbase + L::oQE, ap = sbase + L::oAP;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // [dKBE^T | dQE^T] = KiE^T [dA ; dP]^T
            mma_bf16(tmem, smem_desc_sw128(ki + kk * 2048, 8192, 1024), smem_desc_sw128(ap + kk * 32, 16, 1024),
                     idesc_bf16(128, 128, true, false), kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // dKiE^T = KBE^T dA ...
            mma_bf16(tmem + 128, smem_desc_sw128(kb + kk * 2048, 8192, 1024),
                     smem_desc_sw128(ap + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)  // ... + QE^T dP
            mma_bf16(tmem + 128, smem_desc_sw128(qe + kk * 2048, 8192, 1024),
                     smem_desc_sw128(ap + 8192 + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), 1);
        mma_commit(bar);
        if (!mbar_wait(bar, 0)) {
            fail = 1;
            record_status(GDR_ERR_TIMEOUT);
            mbar_wait(bar, 0);  // the MMAs must be done before TMEM is freed
        }
    }
    tc_before_sync();
    fail = __syncthreads_or(fail);
    tc_after_sync();

    if (!fail) {
        // columns r of this quarter: 0-63 dKBE^T, 64-127 dQE^T, 128-191 dKiE^T
        float akb[RQ], aqe[RQ], aki[RQ];
        if (use_mma) {
            const uint32_t tl = tmem + ((uint32_t)((warp & 3) * 32) << 16) + r0;
            tmem_ld16(tl, akb);
            tmem_ld16(tl + 64, aqe);
            tmem_ld16(tl + 128, aki);
        } else {
#pragma unroll
            for (int i = 0; i < RQ; ++i) akb[i] = aqe[i] = aki[i] = 0.f;
        }
        // per token: the chain rule through the gates; dG (kept in akb) for the suffix sums
        float *dg = akb;
        float g = g0;
#pragma unroll
        for (int i = 0; i < RQ; ++i) {
            const int r = r0 + i;
            float skb = akb[i], sqe = aqe[i], ski = aki[i];
            dg[i] = 0.f;
            if (r >= n) continue;
            const size_t off = (tok0 + (size_t)r * H) * DK + j;
            g += log_alpha[off];
#pragma unroll
            for (int s = 0; s < NS; ++s) {
                skb += part_kb[(size_t)s * BTH * DK + off];
                sqe += part_qe[(size_t)s * BTH * DK + off];
                ski += part_ki[(size_t)s * BTH * DK + off];
            }
            const float e = expf(g), ie = 1.f / e;
            const float kv = to_f32(k[off]), qv = to_f32(q[off]), bv = bgate[off];
            dk[off] = from_f32<Tio>(fmaf(skb * bv, e, ski * ie));
            db[off] = skb * kv * e;
            dq[off] = from_f32<Tio>(sqe * e);
            dg[i] = skb * kv * bv * e + sqe * qv * e - ski * kv * ie;
        }
        // dlog alpha_r = E_C dE_C + sum of dG over tokens r .. n-1 (later quarters first)
        float tot = 0.f;
#pragma unroll
        for (int i = 0; i < RQ; ++i) tot += dg[i];
        __syncthreads();  // every read of `scan` (the gate totals) is done
        scan[rq * DK + j] = tot;
        __syncthreads();
        float dec = 0.f;
#pragma unroll
        for (int s = 0; s < NS; ++s) dec += part_ec[(((size_t)s * nbh + bh) * nchunks + ch) * DK + j];
        float suffix = expf(gC) * dec;  // dG_C, carried by the chunk's last token
#pragma unroll
        for (int u = 3; u > rq; --u) suffix += scan[u * DK + j];
#pragma unroll
        for (int i = RQ - 1; i >= 0; --i) {
            const int r = r0 + i;
            suffix += dg[i];
            if (r < n) dlog_alpha[(tok0 + (size_t)r * H) * DK + j] = suffix;
        }
    } else {
        __syncthreads();
        __syncthreads();
    }
    tc_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 256);
    }
}

// One CTA per (b*H + h, chunk).
template <typename Tio, int NS>
__global__ void __launch_bounds__(kBwd2TcThreads, 1)
gdr2_bwd_chunk_tc_kernel(int T, int H, const Tio *__restrict__ q, const Tio *__restrict__ k,
                         const float *__restrict__ log_alpha, const float *__restrict__ bgate,
                         const float *__restrict__ part_kb, const float *__restrict__ part_qe,
                         const float *__restrict__ part_ki, const float *__restrict__ part_ec,
                         const float *__restrict__ part_x, const int *__restrict__ exact_flags,
                         const float *__restrict__ dAP, Tio *__restrict__ dq, Tio *__restrict__ dk,
                         float *__restrict__ dlog_alpha, float *__restrict__ db, size_t BTH) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    gdr2_bwd_chunk_tc_body<Tio, NS>(T, H, q, k, log_alpha, bgate, part_kb, part_qe, part_ki, part_ec, part_x,
                                    exact_flags, dAP, dq, dk, dlog_alpha, db, BTH, (int)(blockIdx.x / nchunks),
                                    (int)(blockIdx.x % nchunks));
}

// The chunks in todo[0 .. *ntodo) (each b*H*nchunks + chunk): CTA g takes
// items g, g + gridDim.x, ...
template <typename Tio, int NS>
__global__ void __launch_bounds__(kBwd2TcThreads, 1)
gdr2_bwd_chunk_tc_list_kernel(int T, int H, const Tio *__restrict__ q, const Tio *__restrict__ k,
                              const float *__restrict__ log_alpha, const float *__restrict__ bgate,
                              const float *__restrict__ part_kb, const float *__restrict__ part_qe,
                              const float *__restrict__ part_ki, const float *__restrict__ part_ec,
                              const float *__restrict__ part_x, const int *__restrict__ exact_flags,
                              const float *__restrict__ dAP, Tio *__restrict__ dq, Tio *__restrict__ dk,
                              float *__restrict__ dlog_alpha, float *__restrict__ db, size_t BTH,
                              const int *__restrict__ todo, const int *__restrict__ ntodo) {
    const int nchunks = (T + kChunk - 1) / kChunk, n_items = *ntodo;
#pragma unroll 1
    for (int it = blockIdx.x; it < n_items; it += gridDim.x) {
        __syncthreads();  // the previous item is done with shared memory and TMEM
        const int tile = todo[it];
        gdr2_bwd_chunk_tc_body<Tio, NS>(T, H, q, k, log_alpha, bgate, part_kb, part_qe, part_ki, part_ec, part_x,
                                        exact_flags, dAP, dq, dk, dlog_alpha, db, BTH, tile / nchunks,
                                        tile % nchunks);
    }
}

}  // namespace gdr
