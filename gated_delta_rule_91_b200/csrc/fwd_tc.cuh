// fwd_tc.cuh -- chunkwise forward on the 5th-generation tensor cores
// (tcgen05 + TMEM + TMA), bf16 q/k/v/o, dk = dv = 128, fp32 state.
//
// Same chunk algebra as fwd_simt.cuh (Gated DeltaNet review,
// meaningful96.github.io/nr/GDN, section 3.7, UT transform / WY form, with
// the decayed intra-chunk mask and W = T diag(beta gamma) K):
//     A   = strictLower(diag(beta)(Gamma * K K^T)),  T = (I + A)^{-1}
//     U^g = T diag(beta) V,   W = T diag(beta gamma) K,   U = U^g - W S^T
//     O   = diag(gamma) Q S^T + (Q K^T * L) U
//     S'  = gamma_C S + U^T diag(exp(g_C - g)) K
// Every dense product runs as tcgen05.mma with M = 128 by putting the head
// dimension on M (the transposed products):
//     [K;Q] K^T      M=128 (64 K rows + 64 Q rows)  N=64   K=dk    -> K K^T, Q K^T
//     W^T = K^T T''^T     M=dk   N=64  K=64    (T'' = T diag(beta gamma))
//     U^T = V^T T'^T      M=dv   N=64  K=64    (T'  = T diag(beta))
//     O1^T = S Q^T        M=dv   N=64  K=dk
//     U^T -= S W^T        M=dv   N=64  K=dk    (B negated in the descriptor)
//     O2^T = U^T P^T      M=dv   N=64  K=64    (P = Q K^T * L)
//     S   += U~^T K       M=dv   N=dk  K=64    (U~ = diag(exp(g_C - g)) U; S pre-scaled by gamma_C)
// so the fp32 state lives in TMEM (128 lanes x 128 columns) for the whole
// sequence, thread t of the CTA owns TMEM lane t (state row t), and
// O = diag(gamma) O1 + O2 is formed in the epilogue.  The 64 x 64 unit lower
// triangular inverse T is computed on CUDA cores in fp32 (16 x 16 diagonal
// blocks by substitution, off-diagonal blocks by block forward substitution).
//
// Q, K, V tiles (64 tokens x 128) arrive by TMA (128B swizzle, no
// multicast) into a 2-stage ring, so the next chunk's tiles load while the
// current chunk computes; tokens past T are zero-filled by the tensor map.
// One CTA per (b, h), 128 threads.  Thread 0 issues TMA and MMA; every
// mbarrier wait is bounded and a timeout aborts the CTA cleanly (status word
// GDR_ERR_TIMEOUT), waiting for its in-flight copies and freeing TMEM.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "sm100.cuh"

namespace gdr {

constexpr int kTcThreads = 128;

struct FwdTcSmem {
    static constexpr uint32_t KQ_HALF = 128 * 128;  // one dk half: rows 0-63 K, 64-127 Q (16 KB)
    static constexpr uint32_t KQ_STAGE = 2 * KQ_HALF;
    static constexpr uint32_t V_HALF = 64 * 128;    // one dv half: 64 token rows (8 KB)
    static constexpr uint32_t V_STAGE = 2 * V_HALF;
    static constexpr uint32_t oKQ = 0;                        // 2 stages
    static constexpr uint32_t oV = oKQ + 2 * KQ_STAGE;        // 2 stages
    static constexpr uint32_t oP = oV + 2 * V_STAGE;          // P      [r][i]    K-major, 8 KB
    static constexpr uint32_t oT1 = oP + 8192;                // T'     [r][i]    K-major, 8 KB
    static constexpr uint32_t oT2 = oT1 + 8192;               // T''    [r][i]    K-major, 8 KB
    static constexpr uint32_t oW = oT2 + 8192;                // W      [j][r]    MN-major, 16 KB
    static constexpr uint32_t oSB = oW + 16384;               // S bf16 [c][j]    K-major, 32 KB
    static constexpr uint32_t oU = oSB;                       //   aliased later: U^T  [c][r] 16 KB
    static constexpr uint32_t oUt = oSB + 16384;              //                  U~^T [c][r] 16 KB
    static constexpr uint32_t oA = oSB + 32768;               // fp32 A  64 x 68
    static constexpr uint32_t oT = oA + 64 * 68 * 4;          // fp32 T  64 x 68
    static constexpr uint32_t oGate = oT + 64 * 68 * 4;       // g, gamma, beta, dec (4 x 64 fp32)
    static constexpr uint32_t oBar = oGate + 4 * 64 * 4;      // 3 mbarriers, tmem slot, abort flag
    static constexpr uint32_t kBytes = oBar + 64;
    static constexpr uint32_t kAlloc = kBytes + 1024;         // + alignment slack
};

// TMEM column map (512 columns allocated)
constexpr uint32_t kTmS = 0, kTmKQ = 128, kTmW = 192, kTmU = 256, kTmO1 = 320, kTmO2 = 384;

// Row stride (floats) of the fp32 64 x 64 matrices A and T: rows start on
// 16-byte boundaries (vector loads) and 68 = 4 mod 32 spreads rows over banks.
constexpr int kLdT = 68;

// T = (I + A)^{-1} for strictly lower 64 x 64 A (fp32, row stride kLdT), with
// 128 threads, by recursive doubling: 16 x 16 diagonal inverses by
// substitution, then [[T1,0],[L21,T2]]^-1 = [[T1,0],[-T2 L21 T1, T2]] at the
// 32 and 64 levels.  Only the lower triangle (incl. diagonal) of T is
// meaningful.  The upper triangle of A holds the intermediate products.
__device__ __forceinline__ void invert_unit_lower_64(float *sA, float *sT) {
    constexpr int LD = kLdT;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    {   // zero T[0:16,16:32] and T[32:48,48:64] (upper parts of the 32-blocks)
        const int idx = tid * 4, blk = idx >> 8, e = idx & 255;
        float4 *p = reinterpret_cast<float4 *>(sT + (blk * 32 + (e >> 4)) * LD + blk * 32 + 16 + (e & 15));
        *p = make_float4(0.f, 0.f, 0.f, 0.f);
    }
    if (lane < 16) {  // 16 x 16 diagonal block `warp`, column `lane`
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
    // 32 level: for P in {0,1}: X = A[32P+16:32P+32, 32P:32P+16] t_{2P};  T21 = -t_{2P+1} X
    {
        const int P = tid >> 6, rr = (tid & 63) >> 2, cq = (tid & 3) * 4, o = 32 * P;
        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float a = sA[(o + 16 + rr) * LD + o + k];
            const float4 t4 = *reinterpret_cast<const float4 *>(sT + (o + k) * LD + o + cq);
            acc.x = fmaf(a, t4.x, acc.x); acc.y = fmaf(a, t4.y, acc.y);
            acc.z = fmaf(a, t4.z, acc.z); acc.w = fmaf(a, t4.w, acc.w);
        }
        *reinterpret_cast<float4 *>(sA + (o + rr) * LD + o + 16 + cq) = acc;  // X parked above the diagonal
        __syncthreads();
        acc = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            const float t = sT[(o + 16 + rr) * LD + o + 16 + k];
            const float4 x4 = *reinterpret_cast<const float4 *>(sA + (o + k) * LD + o + 16 + cq);
            acc.x = fmaf(t, x4.x, acc.x); acc.y = fmaf(t, x4.y, acc.y);
            acc.z = fmaf(t, x4.z, acc.z); acc.w = fmaf(t, x4.w, acc.w);
        }
        *reinterpret_cast<float4 *>(sT + (o + 16 + rr) * LD + o + cq) =
            make_float4(-acc.x, -acc.y, -acc.z, -acc.w);
        __syncthreads();
    }
    // 64 level: X = A[32:64, 0:32] T[0:32, 0:32];  T[32:64, 0:32] = -T[32:64, 32:64] X
    {
        const int r0 = (tid >> 3) * 2, cq = (tid & 7) * 4;
        float4 acc0 = make_float4(0.f, 0.f, 0.f, 0.f), acc1 = acc0;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float a0 = sA[(32 + r0) * LD + k], a1 = sA[(33 + r0) * LD + k];
            const float4 t4 = *reinterpret_cast<const float4 *>(sT + k * LD + cq);
            acc0.x = fmaf(a0, t4.x, acc0.x); acc0.y = fmaf(a0, t4.y, acc0.y);
            acc0.z = fmaf(a0, t4.z, acc0.z); acc0.w = fmaf(a0, t4.w, acc0.w);
            acc1.x = fmaf(a1, t4.x, acc1.x); acc1.y = fmaf(a1, t4.y, acc1.y);
            acc1.z = fmaf(a1, t4.z, acc1.z); acc1.w = fmaf(a1, t4.w, acc1.w);
        }
        *reinterpret_cast<float4 *>(sA + r0 * LD + 32 + cq) = acc0;        // X parked in A[0:32, 32:64]
        *reinterpret_cast<float4 *>(sA + (r0 + 1) * LD + 32 + cq) = acc1;
        __syncthreads();
        acc0 = make_float4(0.f, 0.f, 0.f, 0.f);
        acc1 = acc0;
#pragma unroll 8
        for (int k = 0; k < 32; ++k) {
            const float t0 = sT[(32 + r0) * LD + 32 + k], t1 = sT[(33 + r0) * LD + 32 + k];
            const float4 x4 = *reinterpret_cast<const float4 *>(sA + k * LD + 32 + cq);
            acc0.x = fmaf(t0, x4.x, acc0.x); acc0.y = fmaf(t0, x4.y, acc0.y);
            acc0.z = fmaf(t0, x4.z, acc0.z); acc0.w = fmaf(t0, x4.w, acc0.w);
            acc1.x = fmaf(t1, x4.x, acc1.x); acc1.y = fmaf(t1, x4.y, acc1.y);
            acc1.z = fmaf(t1, x4.z, acc1.z); acc1.w = fmaf(t1, x4.w, acc1.w);
        }
        *reinterpret_cast<float4 *>(sT + (32 + r0) * LD + cq) = make_float4(-acc0.x, -acc0.y, -acc0.z, -acc0.w);
        *reinterpret_cast<float4 *>(sT + (33 + r0) * LD + cq) = make_float4(-acc1.x, -acc1.y, -acc1.z, -acc1.w);
        __syncthreads();
    }
}

__global__ void __launch_bounds__(kTcThreads, 1)
gdr_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                  const __grid_constant__ CUtensorMap tm_v, int T, int H,
                  const float *__restrict__ log_alpha, const float *__restrict__ beta,
                  const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o,
                  float *__restrict__ S_T) {
    using L = FwdTcSmem;
    using namespace sm100;
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5;
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int nch = (T + kChunk - 1) / kChunk;

    uint64_t *tma_bar = reinterpret_cast<uint64_t *>(sm + L::oBar);  // [2]
    uint64_t *mma_bar = tma_bar + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_bar + 3);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *sg = reinterpret_cast<float *>(sm + L::oGate);
    float *sgam = sg + 64, *sbeta = sg + 128, *sdec = sg + 192;
    float *sA = reinterpret_cast<float *>(sm + L::oA);
    float *sT = reinterpret_cast<float *>(sm + L::oT);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(&tma_bar[0], 1);
        mbar_init(&tma_bar[1], 1);
        mbar_init(mma_bar, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);  // this warp's TMEM lane quarter

    // entry state -> TMEM (row tid)
    {
        float v[32];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            if (S0) {
                const float4 *src = reinterpret_cast<const float4 *>(S0 + ((size_t)bh * D + tid) * D + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 x = src[i];
                    v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
                }
            } else {
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] = 0.f;
            }
            tmem_st32(tl + kTmS + c * 32, v);
        }
        tmem_wait_st();
    }

    auto issue_tma = [&](int n, int s) {
        uint8_t *kq = sm + L::oKQ + s * L::KQ_STAGE;
        uint8_t *vv = sm + L::oV + s * L::V_STAGE;
        mbar_expect_tx(&tma_bar[s], L::KQ_STAGE + L::V_STAGE);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(kq + half * L::KQ_HALF, &tm_k, &tma_bar[s], half * 64, h, n * kChunk, b);
            tma_load_4d(kq + half * L::KQ_HALF + 64 * 128, &tm_q, &tma_bar[s], half * 64, h, n * kChunk, b);
            tma_load_4d(vv + half * L::V_HALF, &tm_v, &tma_bar[s], half * 64, h, n * kChunk, b);
        }
    };
    if (tid == 0) issue_tma(0, 0);

    uint32_t mma_phase = 0;
    int tma_issued = 1, tma_done = 0;  // tracked by thread 0 for the abort path

    // one MMA group completion (thread 0 waits, everyone syncs)
    auto mma_sync_point = [&]() {
        if (tid == 0) {
            mma_commit(mma_bar);
            if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        }
        mma_phase ^= 1;
        __syncthreads();
        tc_after_sync();
    };

#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        const int s = n & 1;
        const int c0 = n * kChunk, nv = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        __syncthreads();  // previous chunk's epilogue is done with the gate arrays
        if (*abort_flag) break;
        if (tid == 0 && n + 1 < nch) {
            issue_tma(n + 1, s ^ 1);
            ++tma_issued;
        }
        if (warp == 0) {  // gates: g (inclusive prefix sum), gamma, beta, exp(g_C - g)
            const int lane = tid;
            const int r0 = 2 * lane, r1 = r0 + 1;
            const float l0 = r0 < nv ? log_alpha[tok0 + (size_t)r0 * H] : 0.f;
            const float l1 = r1 < nv ? log_alpha[tok0 + (size_t)r1 * H] : 0.f;
            float incl = l0 + l1;
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_up_sync(0xffffffffu, incl, off);
                if (lane >= off) incl += y;
            }
            const float g1 = incl, g0 = incl - l1;
            const float gC = __shfl_sync(0xffffffffu, incl, 31);
            sg[r0] = g0; sg[r1] = g1;
            sgam[r0] = expf(g0); sgam[r1] = expf(g1);
            sdec[r0] = expf(gC - g0); sdec[r1] = expf(gC - g1);
            sbeta[r0] = r0 < nv ? beta[tok0 + (size_t)r0 * H] : 0.f;
            sbeta[r1] = r1 < nv ? beta[tok0 + (size_t)r1 * H] : 0.f;
        }
        if (tid == 0) {
            if (!mbar_wait(&tma_bar[s], (uint32_t)((n >> 1) & 1))) *abort_flag = 1;
            else ++tma_done;
        }
        __syncthreads();
        if (*abort_flag) break;

        const uint32_t kq = sbase + L::oKQ + s * L::KQ_STAGE;
        const uint32_t vt = sbase + L::oV + s * L::V_STAGE;

        // ---- MMA 1: [K;Q] K^T -> TMEM KQ (lanes 0-63: K K^T, 64-127: Q K^T) ----
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint32_t a = kq + (kk >> 2) * L::KQ_HALF + (kk & 3) * 32;
                const uint64_t d = smem_desc_sw128(a, 16, 1024);
                mma_bf16(tmem + kTmKQ, d, d, idesc_bf16(128, 64, false, false), kk > 0);
            }
        }
        mma_sync_point();
        if (*abort_flag) break;

        // ---- A (fp32, rows 0-63) and P (bf16 K-major, rows 64-127) ----
        {
            float v[64];
            tmem_ld32(tl + kTmKQ, v);
            tmem_ld32(tl + kTmKQ + 32, v + 32);
            if (tid < 64) {
                const int r = tid;
                const float gr = sg[r], br = sbeta[r];
#pragma unroll
                for (int i = 0; i < 64; ++i)
                    sA[r * kLdT + i] = (i < r) ? br * expf(gr - sg[i]) * v[i] : 0.f;
            } else {
                const int r = tid - 64;
                const float gr = sg[r];
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] = (i <= r) ? expf(gr - sg[i]) * v[i] : 0.f;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::oP + sw128_offset(r, ch), v + 8 * ch);
            }
        }
        __syncthreads();
        invert_unit_lower_64(sA, sT);

        // ---- T' = T diag(beta), T'' = T diag(beta gamma) (bf16 K-major) ; S -> bf16, S *= gamma_C ----
        {
            const int r = tid & 63;
            const bool second = tid >= 64;
            float v[8];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = ch * 8 + e;
                    const float t = (i <= r) ? sT[r * kLdT + i] : 0.f;
                    v[e] = t * sbeta[i] * (second ? sgam[i] : 1.f);
                }
                st_bf16x8(sm + (second ? L::oT2 : L::oT1) + sw128_offset(r, ch), v);
            }
        }
        {
            const float gC = sgam[kChunk - 1];
            float v[32];
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                tmem_ld32(tl + kTmS + c * 32, v);
                uint8_t *half = sm + L::oSB + (c >> 1) * 16384;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4)
                    st_bf16x8(half + sw128_offset(tid, (c & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= gC;
                tmem_st32(tl + kTmS + c * 32, v);
            }
            tmem_wait_st();
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // ---- MMA 2, 3 and O1 ----
        if (tid == 0) {
            tc_after_sync();
            const uint32_t t1 = sbase + L::oT1, t2 = sbase + L::oT2, sb = sbase + L::oSB;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // W^T = K^T T''^T  (A MN-major)
                const uint64_t a = smem_desc_sw128(kq + kk * 2048, L::KQ_HALF, 1024);
                const uint64_t bd = smem_desc_sw128(t2 + kk * 32, 16, 1024);
                mma_bf16(tmem + kTmW, a, bd, idesc_bf16(128, 64, true, false), kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // U^gT = V^T T'^T  (A MN-major)
                const uint64_t a = smem_desc_sw128(vt + kk * 2048, L::V_HALF, 1024);
                const uint64_t bd = smem_desc_sw128(t1 + kk * 32, 16, 1024);
                mma_bf16(tmem + kTmU, a, bd, idesc_bf16(128, 64, true, false), kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {  // O1^T = S Q^T
                const uint64_t a = smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t bd =
                    smem_desc_sw128(kq + (kk >> 2) * L::KQ_HALF + 64 * 128 + (kk & 3) * 32, 16, 1024);
                mma_bf16(tmem + kTmO1, a, bd, idesc_bf16(128, 64, false, false), kk > 0);
            }
        }
        mma_sync_point();
        if (*abort_flag) break;

        // ---- W (bf16, MN-major B operand: row j holds W[0..63][j]) ----
        {
            float v[64];
            tmem_ld32(tl + kTmW, v);
            tmem_ld32(tl + kTmW + 32, v + 32);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::oW + sw128_offset(tid, ch), v + 8 * ch);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // ---- MMA 4: U^T -= S W^T ----
        if (tid == 0) {
            tc_after_sync();
            const uint32_t sb = sbase + L::oSB, w = sbase + L::oW;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const uint64_t a = smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(w + kk * 2048, 8192, 1024);
                mma_bf16(tmem + kTmU, a, bd, idesc_bf16(128, 64, false, true, true), 1);
            }
        }
        mma_sync_point();
        if (*abort_flag) break;

        // ---- U^T and U~^T = U^T diag(exp(g_C - g)) as bf16 K-major A operands ----
        {
            float v[64];
            tmem_ld32(tl + kTmU, v);
            tmem_ld32(tl + kTmU + 32, v + 32);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::oU + sw128_offset(tid, ch), v + 8 * ch);
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] *= sdec[i];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::oUt + sw128_offset(tid, ch), v + 8 * ch);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // ---- MMA 5: O2^T = U^T P^T ; MMA 6: S += U~^T K ----
        if (tid == 0) {
            tc_after_sync();
            const uint32_t u = sbase + L::oU, ut = sbase + L::oUt, p = sbase + L::oP;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_sw128(u + kk * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(p + kk * 32, 16, 1024);
                mma_bf16(tmem + kTmO2, a, bd, idesc_bf16(128, 64, false, false), kk > 0);
            }
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
                const uint64_t a = smem_desc_sw128(ut + kk * 32, 16, 1024);
                const uint64_t bd = smem_desc_sw128(kq + kk * 2048, L::KQ_HALF, 1024);
                mma_bf16(tmem + kTmS, a, bd, idesc_bf16(128, 128, false, true), 1);
            }
        }
        mma_sync_point();
        if (*abort_flag) break;

        // ---- epilogue: O[r][c] = gamma_r O1^T[c][r] + O2^T[c][r] ----
        {
            float v1[32], v2[32];
#pragma unroll 1
            for (int half = 0; half < 2; ++half) {
                tmem_ld32(tl + kTmO1 + half * 32, v1);
                tmem_ld32(tl + kTmO2 + half * 32, v2);
#pragma unroll
                for (int i = 0; i < 32; ++i) {
                    const int r = half * 32 + i;
                    if (r < nv)
                        o[(tok0 + (size_t)r * H) * D + tid] =
                            __float2bfloat16_rn(fmaf(sgam[r], v1[i], v2[i]));
                }
            }
        }
    }

    if (*abort_flag) {
        // drain this CTA's in-flight copies before giving the smem back
        if (tid == 0) {
            record_status(GDR_ERR_TIMEOUT);
            for (int k2 = tma_done; k2 < tma_issued; ++k2) mbar_wait(&tma_bar[k2 & 1], (uint32_t)((k2 >> 1) & 1));
            mma_commit(mma_bar);
            mbar_wait(mma_bar, mma_phase);
        }
    } else if (S_T) {
        float v[32];
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
            tmem_ld32(tl + kTmS + c * 32, v);
            float4 *dst = reinterpret_cast<float4 *>(S_T + ((size_t)bh * D + tid) * D + c * 32);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
    tc_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// ---- host side -------------------------------------------------------------------
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                  const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                  const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

inline EncodeTiledFn encode_tiled_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    }
    return fn;
}

// 4-D map over a [B, T, H, d] bf16 tensor: box = 64 channels x 1 head x 64 tokens x 1 batch,
// 128B swizzle; tokens past T read as zero.
inline bool make_token_map(CUtensorMap *map, const void *base, int B, int T, int H, int d) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 2, (cuuint64_t)H * d * 2, (cuuint64_t)T * H * d * 2};
    const cuuint32_t box[4] = {64, 1, (cuuint32_t)kChunk, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

inline cudaError_t launch_fwd_tc(int B, int T, int H, const void *q, const void *k, const void *v,
                                 const float *la, const float *beta, const float *S0, void *o,
                                 float *S_T, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)FwdTcSmem::kAlloc);
    if (err != cudaSuccess) return err;
    gdr_fwd_tc_kernel<<<(unsigned)(B * H), kTcThreads, FwdTcSmem::kAlloc, stream>>>(
        mq, mk, mv, T, H, la, beta, S0, static_cast<__nv_bfloat16 *>(o), S_T);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
