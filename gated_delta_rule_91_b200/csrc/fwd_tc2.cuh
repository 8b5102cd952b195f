// fwd_tc2.cuh -- chunkwise forward on tcgen05, split over a 2-CTA cluster
// per (b, h): a "prep" CTA and a "state" CTA on two SMs, 512 threads each.
//
// Same chunk algebra and operand orientation as fwd_tc.cuh (Gated DeltaNet
// review, meaningful96.github.io/nr/GDN, section 3.7: UT transform / WY form
// with the decayed intra-chunk mask and W = T diag(beta gamma) K).  The work
// that does not depend on the state S runs one chunk ahead on its own SM:
//
//   prep CTA (rank 0), per chunk n:
//     [K;Q] K^T (tcgen05, M=128)  ->  A = strictLower(diag(beta) Gamma*KK^T) (fp32),
//                                     P = (Q K^T) * L                       (bf16)
//     T = (I + A)^{-1} (fp32, CUDA cores), T' = T diag(beta), T'' = T diag(beta gamma)
//     Q~ = diag(gamma) Q,  gates gamma_r and exp(g_C - g_r)
//     -> one DSMEM bulk copy (41.5 KB) into the state CTA's slot n % 2
//   state CTA (rank 1), per chunk n (fp32 S resident in TMEM):
//     W^T = K^T T''^T, U^gT = V^T T'^T       (issued one chunk ahead)
//     U^T -= S W^T,  O^T = S Q~^T           (S read as bf16 operand)
//     O^T += U^T P^T,  S = gamma_C S + U~^T K
//     O staged in shared memory and written by a TMA store.
// The decay ratio exp(g_r - g_i) of the masks is formed as
// gamma'_r * (1/gamma'_i) with gamma' = exp(g - g_31) taken about the chunk's
// middle token (two multiplies per element, no exponential); a chunk whose
// decay range exceeds e^80 (where those factors could overflow) takes the
// exact per-element exponential instead.
//
// Warp w of each CTA owns TMEM lane quarter w % 4 and column group w / 4 (of
// four); thread 0 issues TMA and MMA.  Sixteen warps (four per SM
// sub-partition) hide the latency of the CUDA-core phases, each written as
// vector loads, then arithmetic, then vector stores.  The prep waits for a free hand-off
// slot only after the inverse, so the state CTA's tail overlaps it.  Slots go
// back to the prep CTA with a remote mbarrier arrive.  No TMA multicast; each
// CTA loads its own tiles (the shared K/Q tiles hit L2 for the second reader).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "fwd_tc.cuh"
#include "sm100.cuh"

namespace gdr {

constexpr int kTc2Threads = 512;

struct Tc2Layout {
    // hand-off slot (identical offsets in the prep staging area and the state slots)
    static constexpr uint32_t H_T1 = 0;       // T'   [r][i]  K-major bf16, 8 KB
    static constexpr uint32_t H_T2 = 8192;    // T''  [r][i]  K-major bf16, 8 KB
    static constexpr uint32_t H_P = 16384;    // P    [r][i]  K-major bf16, 8 KB
    static constexpr uint32_t H_QT = 24576;   // Q~   [r][j]  K-major bf16, 2 halves x 8 KB
    static constexpr uint32_t H_G = 40960;    // gamma[64], dec[64] fp32
    static constexpr uint32_t H_BYTES = 40960 + 512;
    static constexpr uint32_t H_SLOT = 41984;  // 41 KB: keeps every slot 1024-aligned
    // state CTA
    static constexpr uint32_t S_K = 0;                    // 2 stages x (2 halves x 64 rows x 128 B)
    static constexpr uint32_t S_V = S_K + 2 * 16384;
    static constexpr uint32_t S_H = S_V + 2 * 16384;      // 2 hand-off slots
    static constexpr uint32_t S_W = S_H + 2 * H_SLOT;     // W [j][r] MN-major, 16 KB
    static constexpr uint32_t S_SB = S_W + 16384;         // S bf16 [c][j] (32 KB); later U^T, U~^T
    static constexpr uint32_t S_OST = S_SB + 32768;       // O tile for the TMA store, 2 halves x 8 KB
    static constexpr uint32_t S_GL = S_OST + 16384;       // gamma of chunks by parity: [2][64] fp32
    static constexpr uint32_t S_BAR = S_GL + 512;
    static constexpr uint32_t S_BYTES = S_BAR + 128;
    // prep CTA
    static constexpr uint32_t P_KQ = 0;                   // 2 stages x 32 KB ([K;Q] per dk half)
    static constexpr uint32_t P_A = P_KQ + 2 * 32768;
    static constexpr uint32_t P_T = P_A + 64 * kLdT * 4;
    static constexpr uint32_t P_STG = P_T + 64 * kLdT * 4;  // 2 staging slots
    static constexpr uint32_t P_GATE = P_STG + 2 * H_SLOT;  // g, beta, gamma, dec, gamma', 1/gamma' [64] + flag
    static constexpr uint32_t P_BAR = P_GATE + 6 * 256 + 16;
    static constexpr uint32_t P_BYTES = P_BAR + 128;
    static constexpr uint32_t kAlloc = (S_BYTES > P_BYTES ? S_BYTES : P_BYTES) + 1024;
};
static_assert(Tc2Layout::S_H % 1024 == 0 && Tc2Layout::S_W % 1024 == 0 && Tc2Layout::S_SB % 1024 == 0 &&
                  Tc2Layout::S_OST % 1024 == 0,
              "state tiles must be 1024-aligned");
static_assert(Tc2Layout::P_STG % 1024 == 0 && Tc2Layout::H_SLOT % 1024 == 0, "slots must be 1024-aligned");
static_assert(Tc2Layout::kAlloc <= 232448, "shared memory budget");

// state TMEM columns (512 allocated)
constexpr uint32_t kT2S = 0, kT2W = 128, kT2U = 192, kT2O = 320;  // U, O double-buffered (+64)

// T = (I + A)^{-1} for strictly lower 64 x 64 A (fp32, row stride kLdT) with
// 512 threads; same recursive doubling as invert_unit_lower_64 (16 x 16
// diagonal inverses by substitution, then the 32 and 64 levels), retiled for
// sixteen warps.  Only the lower triangle of T is meaningful; the upper
// triangle of A holds the intermediate products.
__device__ __forceinline__ void invert_unit_lower_64_w16(float *sA, float *sT) {
    constexpr int LD = kLdT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    {   // zero T[0:16,16:32] and T[32:48,48:64]
        const int blk = tid >> 8, e = tid & 255;
        sT[(blk * 32 + (e >> 4)) * LD + blk * 32 + 16 + (e & 15)] = 0.f;
    }
    if (warp < 4 && lane < 16) {  // 16 x 16 diagonal block `warp`, column `lane`
        const int base = warp * 16, j = lane;
        float t[16];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            float acc0 = (r == j) ? 1.f : 0.f, acc1 = 0.f;
#pragma unroll
            for (int i = 0; i + 1 < r; i += 2) {
                acc0 = fmaf(-sA[(base + r) * LD + base + i], t[i], acc0);
                acc1 = fmaf(-sA[(base + r) * LD + base + i + 1], t[i + 1], acc1);
            }
            if (r & 1) acc0 = fmaf(-sA[(base + r) * LD + base + r - 1], t[r - 1], acc0);
            t[r] = (r < j) ? 0.f : acc0 + acc1;
        }
#pragma unroll
        for (int r = 0; r < 16; ++r) sT[(base + r) * LD + base + j] = t[r];
    }
    __syncthreads();
    {   // 32 level: X = A[o+16:o+32, o:o+16] t_{2P};  T[o+16:o+32, o:o+16] = -t_{2P+1} X
        const int P = tid >> 8, rr = (tid & 255) >> 4, c = tid & 15, o = 32 * P;
        float a[16], acc = 0.f;
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const float4 x = *reinterpret_cast<const float4 *>(sA + (o + 16 + rr) * LD + o + 4 * k4);
            a[4 * k4] = x.x; a[4 * k4 + 1] = x.y; a[4 * k4 + 2] = x.z; a[4 * k4 + 3] = x.w;
        }
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(a[k], sT[(o + k) * LD + o + c], acc);
        sA[(o + rr) * LD + o + 16 + c] = acc;  // X parked above the diagonal
        __syncthreads();
#pragma unroll
        for (int k4 = 0; k4 < 4; ++k4) {
            const float4 x = *reinterpret_cast<const float4 *>(sT + (o + 16 + rr) * LD + o + 16 + 4 * k4);
            a[4 * k4] = x.x; a[4 * k4 + 1] = x.y; a[4 * k4 + 2] = x.z; a[4 * k4 + 3] = x.w;
        }
        acc = 0.f;
#pragma unroll
        for (int k = 0; k < 16; ++k) acc = fmaf(a[k], sA[(o + k) * LD + o + 16 + c], acc);
        sT[(o + 16 + rr) * LD + o + c] = -acc;
        __syncthreads();
    }
    {   // 64 level: X = A[32:64, 0:32] T[0:32, 0:32];  T[32:64, 0:32] = -T[32:64, 32:64] X
        const int r = tid >> 4, cq = (tid & 15) * 2;
        float2 acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            const float4 a4 = *reinterpret_cast<const float4 *>(sA + (32 + r) * LD + 4 * k4);
            const float a[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float2 t2 = *reinterpret_cast<const float2 *>(sT + (4 * k4 + kk) * LD + cq);
                acc.x = fmaf(a[kk], t2.x, acc.x);
                acc.y = fmaf(a[kk], t2.y, acc.y);
            }
        }
        *reinterpret_cast<float2 *>(sA + r * LD + 32 + cq) = acc;  // X parked in A[0:32, 32:64]
        __syncthreads();
        acc = make_float2(0.f, 0.f);
#pragma unroll
        for (int k4 = 0; k4 < 8; ++k4) {
            const float4 t4 = *reinterpret_cast<const float4 *>(sT + (32 + r) * LD + 32 + 4 * k4);
            const float t[4] = {t4.x, t4.y, t4.z, t4.w};
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const float2 x2 = *reinterpret_cast<const float2 *>(sA + (4 * k4 + kk) * LD + 32 + cq);
                acc.x = fmaf(t[kk], x2.x, acc.x);
                acc.y = fmaf(t[kk], x2.y, acc.y);
            }
        }
        *reinterpret_cast<float2 *>(sT + (32 + r) * LD + cq) = make_float2(-acc.x, -acc.y);
        __syncthreads();
    }
}

// ------------------------------------------------------------------ prep CTA --
__device__ __forceinline__ void tc2_prep(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                         int T, int H, int b, int h, const float *log_alpha,
                                         const float *beta) {
    using L = Tc2Layout;
    using namespace sm100;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *tma_full = reinterpret_cast<uint64_t *>(sm + L::P_BAR);  // [2]
    uint64_t *empty = tma_full + 2;                                      // [2], arrived by the state CTA
    uint64_t *mma_bar = tma_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *sg = reinterpret_cast<float *>(sm + L::P_GATE);
    float *sbeta = sg + 64, *sgam = sg + 128, *sdec = sg + 192, *sgp = sg + 256, *sinv = sg + 320;
    volatile int *exact_flag = reinterpret_cast<volatile int *>(sg + 384);
    float *sA = reinterpret_cast<float *>(sm + L::P_A), *sT = reinterpret_cast<float *>(sm + L::P_T);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(&tma_full[0], 1);
        mbar_init(&tma_full[1], 1);
        mbar_init(&empty[0], 1);
        mbar_init(&empty[1], 1);
        mbar_init(mma_bar, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(tm_q);
        prefetch_tmap(tm_k);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 64);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    cluster_sync();  // both CTAs' barriers are initialised (and the state's slots armed)
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t remote_slot0 = cluster_addr(sm + L::S_H, 1);
    const uint32_t remote_full0 = cluster_addr(sm + L::S_BAR + 16, 1);  // state's hand_full[0]

    auto issue_tma = [&](int n, int s) {
        uint8_t *kq = sm + L::P_KQ + s * 32768;
        mbar_expect_tx(&tma_full[s], 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(kq + half * 16384, tm_k, &tma_full[s], half * 64, h, n * kChunk, b);
            tma_load_4d(kq + half * 16384 + 8192, tm_q, &tma_full[s], half * 64, h, n * kChunk, b);
        }
    };
    auto issue_mma1 = [&](int s) {  // [K;Q] K^T -> TMEM (lanes 0-63 K K^T, 64-127 Q K^T)
        const uint32_t kq = sbase + L::P_KQ + s * 32768;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const uint64_t d = smem_desc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
            mma_bf16(tmem, d, d, idesc_bf16(128, 64, false, false), kk > 0);
        }
        mma_commit(mma_bar);
    };
    // gates of one chunk, held by warp 0 (lane l: rows 2l, 2l+1) between load and use
    float pl0 = 0.f, pl1 = 0.f, pb0 = 0.f, pb1 = 0.f;
    auto load_gates = [&](int n) {
        const int c0 = n * kChunk, nv = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        const int r0 = 2 * lane, r1 = r0 + 1;
        pl0 = r0 < nv ? log_alpha[tok0 + (size_t)r0 * H] : 0.f;
        pl1 = r1 < nv ? log_alpha[tok0 + (size_t)r1 * H] : 0.f;
        pb0 = r0 < nv ? beta[tok0 + (size_t)r0 * H] : 0.f;
        pb1 = r1 < nv ? beta[tok0 + (size_t)r1 * H] : 0.f;
    };
    if (warp == 0) load_gates(0);

    int tma_issued = 0, tma_done = 0;
    uint32_t mma_phase = 0;
    if (tid == 0) {
        issue_tma(0, 0);
        ++tma_issued;
        if (nch > 1) {
            issue_tma(1, 1);
            ++tma_issued;
        }
        if (!mbar_wait(&tma_full[0], 0)) *abort_flag = 1;
        else {
            ++tma_done;
            tc_after_sync();
            issue_mma1(0);
        }
    }

#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        const int s = n & 1;
        uint8_t *stg = sm + L::P_STG + s * L::H_SLOT;
        __syncthreads();
        if (*abort_flag) break;
        if (warp == 0) {  // gates: g (inclusive prefix sum), gamma, dec, gamma' = exp(g - g_31), 1/gamma'
            const int r0 = 2 * lane, r1 = r0 + 1;
            float incl = pl0 + pl1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float g1 = incl, g0 = incl - pl1;
            const float gC = __shfl_sync(0xffffffffu, incl, 31);
            const float gM = __shfl_sync(0xffffffffu, g1, 15);  // g_31
            const float gF = __shfl_sync(0xffffffffu, g0, 0);   // g_0
            sg[r0] = g0; sg[r1] = g1;
            sbeta[r0] = pb0; sbeta[r1] = pb1;
            sgam[r0] = expf(g0); sgam[r1] = expf(g1);
            sdec[r0] = expf(gC - g0); sdec[r1] = expf(gC - g1);
            sgp[r0] = expf(g0 - gM); sgp[r1] = expf(g1 - gM);
            sinv[r0] = expf(gM - g0); sinv[r1] = expf(gM - g1);
            if (lane == 0) *exact_flag = (gF - gC) > 80.f;
            if (n + 1 < nch) load_gates(n + 1);  // prefetch: consumed next chunk
        }
        if (tid == 0 && !mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        mma_phase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();

        // A (fp32, rows 0-63 -> sA) and P (rows 64-127, kept in registers), this
        // thread's 16 columns of its TMEM lane
        const int row = wq * 32 + lane;  // 0..127
        const int c0 = wc * 16;
        float pv[16];
        {
            tmem_ld16(tl + c0, pv);
            const bool exact = *exact_flag;
            float sv[16], gv[16];
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const float4 x = *reinterpret_cast<const float4 *>(sinv + c0 + 4 * k4);
                const float4 y = *reinterpret_cast<const float4 *>(sg + c0 + 4 * k4);
                sv[4 * k4] = x.x; sv[4 * k4 + 1] = x.y; sv[4 * k4 + 2] = x.z; sv[4 * k4 + 3] = x.w;
                gv[4 * k4] = y.x; gv[4 * k4 + 1] = y.y; gv[4 * k4 + 2] = y.z; gv[4 * k4 + 3] = y.w;
            }
            const int r = row & 63;
            const float gr = sg[r], br = row < 64 ? sbeta[r] : 1.f;
            const float f = br * sgp[r];
            const int lim = row < 64 ? r : r + 1;  // strictly lower for A, incl. diagonal for P
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const float d = exact ? br * __expf(gr - gv[i]) : f * sv[i];
                pv[i] = (c0 + i < lim) ? d * pv[i] : 0.f;
            }
            if (row < 64) {
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    *reinterpret_cast<float4 *>(sA + r * kLdT + c0 + 4 * k4) =
                        make_float4(pv[4 * k4], pv[4 * k4 + 1], pv[4 * k4 + 2], pv[4 * k4 + 3]);
            }
        }
        tc_before_sync();
        __syncthreads();
        if (tid == 0 && n + 1 < nch) {  // next chunk's K K^T / Q K^T overlaps this chunk's inverse
            tc_after_sync();
            if (!mbar_wait(&tma_full[s ^ 1], (uint32_t)(((n + 1) >> 1) & 1))) *abort_flag = 1;
            else {
                ++tma_done;
                issue_mma1(s ^ 1);
            }
        }
        invert_unit_lower_64_w16(sA, sT);
        // staging slot s (and the state's slot s) must have been consumed (chunk n-2)
        if (tid == 0 && n >= 2 && !mbar_wait_cluster(&empty[s], (uint32_t)(((n >> 1) - 1) & 1))) *abort_flag = 1;
        __syncthreads();
        if (*abort_flag) break;
        {
            float *hg = reinterpret_cast<float *>(stg + L::H_G);
            if (tid < 64) hg[tid] = sgam[tid];
            else if (tid < 128) hg[tid] = sdec[tid - 64];
            // P rows
            if (row >= 64) {
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    st_bf16x8(stg + L::H_P + sw128_offset(row - 64, wc * 2 + ch), pv + 8 * ch);
            }
            // T' = T diag(beta) (rows 0-63), T'' = T diag(beta gamma) (rows 64-127), 16 columns each
            {
                const int r = tid & 63;
                const bool second = (tid & 64) != 0;
                const int cb = (tid >> 7) * 16;
                float t[16], bv[16], gm[16];
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4) {
                    const float4 x = *reinterpret_cast<const float4 *>(sT + r * kLdT + cb + 4 * k4);
                    const float4 y = *reinterpret_cast<const float4 *>(sbeta + cb + 4 * k4);
                    const float4 z = *reinterpret_cast<const float4 *>(sgam + cb + 4 * k4);
                    t[4 * k4] = x.x; t[4 * k4 + 1] = x.y; t[4 * k4 + 2] = x.z; t[4 * k4 + 3] = x.w;
                    bv[4 * k4] = y.x; bv[4 * k4 + 1] = y.y; bv[4 * k4 + 2] = y.z; bv[4 * k4 + 3] = y.w;
                    gm[4 * k4] = z.x; gm[4 * k4 + 1] = z.y; gm[4 * k4 + 2] = z.z; gm[4 * k4 + 3] = z.w;
                }
#pragma unroll
                for (int i = 0; i < 16; ++i)
                    t[i] = (cb + i <= r) ? t[i] * bv[i] * (second ? gm[i] : 1.f) : 0.f;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    st_bf16x8(stg + (second ? L::H_T2 : L::H_T1) + sw128_offset(r, (cb >> 3) + ch), t + 8 * ch);
            }
            // Q~ = diag(gamma) Q: same swizzled positions as the Q tile
            {
                const uint8_t *qt = sm + L::P_KQ + s * 32768 + 8192;
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const int ci = tid * 2 + e;  // 16-byte chunk 0..1023
                    const int half = ci >> 9;
                    const uint32_t ob = (uint32_t)(ci & 511) * 16;
                    const float g = sgam[ob >> 7];
                    float f[8];
                    load8(reinterpret_cast<const __nv_bfloat16 *>(qt + half * 16384 + ob), f);
#pragma unroll
                    for (int i = 0; i < 8; ++i) f[i] *= g;
                    st_bf16x8(stg + L::H_QT + half * 8192 + ob, f);
                }
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            bulk_copy_to_cluster(remote_slot0 + s * L::H_SLOT, stg, L::H_BYTES, remote_full0 + 8 * s);
            if (n + 2 < nch) {  // K/Q stage s is free: its MMA is done and Q~ has been read
                issue_tma(n + 2, s);
                ++tma_issued;
            }
        }
    }

    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        for (int k2 = tma_done; k2 < tma_issued; ++k2) mbar_wait(&tma_full[k2 & 1], (uint32_t)((k2 >> 1) & 1));
        mma_commit(mma_bar);
        mbar_wait(mma_bar, mma_phase);
    }
    tc_before_sync();
    __syncthreads();
    cluster_sync();  // the state CTA has consumed every copy and sent its last arrive
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 64);
    }
}

// ----------------------------------------------------------------- state CTA --
__device__ __forceinline__ void tc2_state(uint8_t *sm, const CUtensorMap *tm_k, const CUtensorMap *tm_v,
                                          const CUtensorMap *tm_o, int T, int H, int b, int h,
                                          const float *S0, float *S_T, bool store_o, float *S_chunks) {
    using L = Tc2Layout;
    using namespace sm100;
    constexpr int D = 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;  // TMEM lane = row of S / U^T / O^T / W^T
    const int bh = b * H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *tma_full = reinterpret_cast<uint64_t *>(sm + L::S_BAR);  // [2]
    uint64_t *hand_full = tma_full + 2;                                  // [2], filled by the prep CTA
    uint64_t *bar_a = tma_full + 4, *bar_b = tma_full + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_full + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *gl = reinterpret_cast<float *>(sm + L::S_GL);  // [2][64] gamma, by chunk parity
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(&tma_full[0], 1);
        mbar_init(&tma_full[1], 1);
        mbar_init(&hand_full[0], 1);
        mbar_init(&hand_full[1], 1);
        mbar_init(bar_a, 1);
        mbar_init(bar_b, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(tm_k);
        prefetch_tmap(tm_v);
        prefetch_tmap(tm_o);
        mbar_expect_tx(&hand_full[0], L::H_BYTES);  // arm the slots for chunks 0 and 1
        if (nch > 1) mbar_expect_tx(&hand_full[1], L::H_BYTES);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    cluster_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t remote_empty0 = cluster_addr(sm + L::P_BAR + 16, 0);  // prep's empty[0]

    {   // entry state -> TMEM (row `row`, this column group's 32 columns)
        float v[32];
        {
            const int col = wc * 32;
            if (S0) {
                const float4 *src = reinterpret_cast<const float4 *>(S0 + ((size_t)bh * D + row) * D + col);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 x = src[i];
                    v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            tmem_st32(tl + kT2S + col, v);
        }
        tmem_wait_st();
    }

    auto issue_tma = [&](int n, int s) {
        uint8_t *kt = sm + L::S_K + s * 16384, *vt = sm + L::S_V + s * 16384;
        mbar_expect_tx(&tma_full[s], 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(kt + half * 8192, tm_k, &tma_full[s], half * 64, h, n * kChunk, b);
            tma_load_4d(vt + half * 8192, tm_v, &tma_full[s], half * 64, h, n * kChunk, b);
        }
    };
    // W^T = K^T T''^T, U^gT = V^T T'^T for chunk n (thread 0), after its inputs landed
    auto issue_wu = [&](int n) -> bool {
        const int s = n & 1;
        if (!mbar_wait(&tma_full[s], (uint32_t)((n >> 1) & 1))) return false;
        if (!mbar_wait_cluster(&hand_full[s], (uint32_t)((n >> 1) & 1))) return false;
        tc_after_sync();
        const uint32_t kt = sbase + L::S_K + s * 16384, vt = sbase + L::S_V + s * 16384;
        const uint32_t hs = sbase + L::S_H + s * L::H_SLOT;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            mma_bf16(tmem + kT2W, smem_desc_sw128(kt + kk * 2048, 8192, 1024),
                     smem_desc_sw128(hs + L::H_T2 + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false),
                     kk > 0);
        }
#pragma unroll
        for (int kk = 0; kk < 4; ++kk) {
            mma_bf16(tmem + kT2U + 64 * s, smem_desc_sw128(vt + kk * 2048, 8192, 1024),
                     smem_desc_sw128(hs + L::H_T1 + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false),
                     kk > 0);
        }
        mma_commit(bar_b);
        return true;
    };
    // O^T of chunk n (lane = value channel, column = token) -> bf16 tile [token][channel]
    auto stage_o = [&](int n) {
        float v[16];
        tmem_ld16(tl + kT2O + 64 * (n & 1) + wc * 16, v);
        uint8_t *half = sm + L::S_OST + (row >> 6) * 8192;
        const int cc = row & 63;
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = wc * 16 + i;
            *reinterpret_cast<__nv_bfloat16 *>(half + sw128_offset(r, cc >> 3) + (cc & 7) * 2) =
                __float2bfloat16_rn(v[i]);
        }
        fence_async_smem();
    };
    auto store_o_tile = [&](int n) {  // thread 0, after a barrier that follows stage_o
        tma_store_4d(tm_o, sm + L::S_OST, 0, h, n * kChunk, b);
        tma_store_4d(tm_o, sm + L::S_OST + 8192, 64, h, n * kChunk, b);
        bulk_commit();
    };
    auto stash_gamma = [&](int n) {  // keep gamma of chunk n after its slot is released
        if (tid < 64) gl[64 * (n & 1) + tid] =
            reinterpret_cast<const float *>(sm + L::S_H + (n & 1) * L::H_SLOT + L::H_G)[tid];
    };

    int tma_issued = 0, tma_done_n = 0;
    uint32_t aphase = 0, bphase = 0;
    if (tid == 0) {
        issue_tma(0, 0);
        ++tma_issued;
        if (nch > 1) {
            issue_tma(1, 1);
            ++tma_issued;
        }
        if (!issue_wu(0)) *abort_flag = 1;
        else if (!mbar_wait(bar_b, bphase)) *abort_flag = 1;
        else tma_done_n = 1;
    }
    bphase ^= 1;
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    if (!*abort_flag) {
        float v[16];
        tmem_ld16(tl + kT2W + wc * 16, v);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::S_W + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
        stash_gamma(0);
        fence_async_smem();
    }
    tc_before_sync();
    __syncthreads();

    int n_done = 0;  // chunks whose MMAs all completed
#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        if (*abort_flag) break;
        const int s = n & 1;
        const uint32_t hs = sbase + L::S_H + s * L::H_SLOT;
        const float *hgate = reinterpret_cast<const float *>(sm + L::S_H + s * L::H_SLOT + L::H_G);

        // (a) S -> bf16 operand; S *= gamma_C (the state update accumulates on top)
        {
            const float gC = gl[64 * s + kChunk - 1];
            float v[32];
            {
                const int col = wc * 32;
                tmem_ld32(tl + kT2S + col, v);
                if (S_chunks) {  // entry state of chunk n, for the backward's recompute
                    float4 *dst = reinterpret_cast<float4 *>(
                        S_chunks + (((size_t)bh * nch + n) * D + row) * D + col);
#pragma unroll
                    for (int i = 0; i < 8; ++i)
                        dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
                }
                uint8_t *half = sm + L::S_SB + (wc >> 1) * 16384;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) st_bf16x8(half + sw128_offset(row, (wc & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= gC;
                tmem_st32(tl + kT2S + col, v);
            }
            tmem_wait_st();
        }
        fence_async_smem();
        if (tid == 0) bulk_wait_read_all();  // the O tile of chunk n-2 has left shared memory
        tc_before_sync();
        __syncthreads();

        // (b) U^T -= S W^T ; O^T = S Q~^T
        if (tid == 0) {
            tc_after_sync();
            const uint32_t sb = sbase + L::S_SB, w = sbase + L::S_W;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t a = smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                mma_bf16(tmem + kT2U + 64 * s, a, smem_desc_sw128(w + kk * 2048, 8192, 1024),
                         idesc_bf16(128, 64, false, true, true), 1);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t a = smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(hs + L::H_QT + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024);
                mma_bf16(tmem + kT2O + 64 * s, a, bd, idesc_bf16(128, 64, false, false), kk > 0);
            }
            mma_commit(bar_a);
        }
        __syncwarp();
        // (c) stage the previous chunk's output, then W/U^g of the next chunk
        if (store_o && n > 0) stage_o(n - 1);
        if (tid == 0 && n + 1 < nch) {
            if (!issue_wu(n + 1)) *abort_flag = 1;
            else ++tma_done_n;
        }
        __syncwarp();
        // (d) U^T, U~^T = U^T diag(exp(g_C - g)) -> bf16 A operands
        if (tid == 0 && !mbar_wait(bar_a, aphase)) *abort_flag = 1;
        aphase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        if (tid == 0 && store_o && n > 0) store_o_tile(n - 1);
        {
            float v[16];
            tmem_ld16(tl + kT2U + 64 * s + wc * 16, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::S_SB + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const float4 dv4 = *reinterpret_cast<const float4 *>(hgate + 64 + wc * 16 + 4 * k4);
                v[4 * k4] *= dv4.x; v[4 * k4 + 1] *= dv4.y; v[4 * k4 + 2] *= dv4.z; v[4 * k4 + 3] *= dv4.w;
            }
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
                st_bf16x8(sm + L::S_SB + 16384 + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // (e) O^T += U^T P^T ; S += U~^T K
        if (tid == 0) {
            tc_after_sync();
            const uint32_t u = sbase + L::S_SB, ut = sbase + L::S_SB + 16384;
            const uint32_t kt = sbase + L::S_K + s * 16384;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kT2O + 64 * s, smem_desc_sw128(u + kk * 32, 16, 1024),
                         smem_desc_sw128(hs + L::H_P + kk * 32, 16, 1024), idesc_bf16(128, 64, false, false), 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kT2S, smem_desc_sw128(ut + kk * 32, 16, 1024),
                         smem_desc_sw128(kt + kk * 2048, 8192, 1024), idesc_bf16(128, 128, false, true), 1);
            mma_commit(bar_a);
            if (n + 1 < nch && !mbar_wait(bar_b, bphase)) *abort_flag = 1;
        }
        if (n + 1 < nch) bphase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        // (f) W of the next chunk -> MN-major B operand (W buffer free: its MMA is done)
        if (n + 1 < nch) {
            float v[16];
            tmem_ld16(tl + kT2W + wc * 16, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::S_W + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
            stash_gamma(n + 1);
            fence_async_smem();
        }
        // (g) chunk n finished: release its hand-off slot and K/V stage
        if (tid == 0) {
            if (!mbar_wait(bar_a, aphase)) *abort_flag = 1;
            else {
                n_done = n + 1;
                if (n + 2 < nch) {
                    mbar_expect_tx(&hand_full[s], L::H_BYTES);
                    mbar_arrive_remote(remote_empty0 + 8 * s);
                    issue_tma(n + 2, s);
                    ++tma_issued;
                }
            }
        }
        aphase ^= 1;
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
    }

    if (!*abort_flag && nch > 0) {
        if (store_o) {
            if (tid == 0) bulk_wait_read_all();
            __syncthreads();
            stage_o(nch - 1);
            __syncthreads();
            if (tid == 0) store_o_tile(nch - 1);
        }
        if (S_T) {
            float v[32];
            {
                const int col = wc * 32;
                tmem_ld32(tl + kT2S + col, v);
                float4 *dst = reinterpret_cast<float4 *>(S_T + ((size_t)bh * D + row) * D + col);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }
    if (tid == 0) bulk_wait_all();  // output stores complete before the CTA exits
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        // drain: this CTA's TMA loads, its MMAs, and the prep CTA's copies into it
        for (int k2 = tma_done_n; k2 < tma_issued; ++k2) mbar_wait(&tma_full[k2 & 1], (uint32_t)((k2 >> 1) & 1));
        mma_commit(bar_a);
        mbar_wait(bar_a, aphase);
        for (int k2 = n_done; k2 < nch && k2 < n_done + 2; ++k2)
            mbar_wait_cluster(&hand_full[k2 & 1], (uint32_t)((k2 >> 1) & 1));
    }
    tc_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTc2Threads, 1)
gdr_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   int T, int H, const float *__restrict__ log_alpha, const float *__restrict__ beta,
                   const float *__restrict__ S0, float *__restrict__ S_T, int store_o,
                   float *__restrict__ S_chunks) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int bh = blockIdx.x >> 1, b = bh / H, h = bh % H;
    if (sm100::cluster_ctarank() == 0)
        tc2_prep(sm, &tm_q, &tm_k, T, H, b, h, log_alpha, beta);
    else
        tc2_state(sm, &tm_k, &tm_v, &tm_o, T, H, b, h, S0, S_T, store_o != 0, S_chunks);
}

// o == nullptr runs the recurrence without writing outputs (the backward's
// recompute); S_chunks (nullable) receives every chunk's entry state,
// [B, H, nchunks, 128, 128] fp32.
inline cudaError_t launch_fwd_tc2(int B, int T, int H, const void *q, const void *k, const void *v,
                                  const float *la, const float *beta, const float *S0, void *o,
                                  float *S_T, cudaStream_t stream, float *S_chunks = nullptr) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128) || !make_token_map(&mo, o ? o : q, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr_fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)Tc2Layout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr_fwd_tc2_kernel<<<(unsigned)(2 * B * H), kTc2Threads, Tc2Layout::kAlloc, stream>>>(
        mq, mk, mv, mo, T, H, la, beta, S0, S_T, o != nullptr ? 1 : 0, S_chunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
