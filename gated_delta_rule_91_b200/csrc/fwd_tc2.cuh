// fwd_tc2.cuh -- chunkwise forward on tcgen05, split over a 2-CTA cluster
// per (b, h): a "prep" CTA and a "state" CTA on two SMs.
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
// so the state CTA's critical path per chunk is: S -> bf16 operand, two MMA
// groups and one U round trip; the epilogue of chunk n-1 and the W/U^g
// products of chunk n+1 overlap its MMAs (double-buffered U and O
// accumulators).  Hand-off slots are released back to the prep CTA with a
// remote mbarrier arrive.  No TMA multicast anywhere; each CTA loads its own
// tiles (the shared K/Q tiles hit L2 for the second reader).
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "fwd_tc.cuh"
#include "sm100.cuh"

namespace gdr {

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
    static constexpr uint32_t S_GL = S_SB + 32768;        // gamma of chunks n, n-1: [2][64] fp32
    static constexpr uint32_t S_BAR = S_GL + 512;
    static constexpr uint32_t S_BYTES = S_BAR + 128;
    // prep CTA
    static constexpr uint32_t P_KQ = 0;                   // 2 stages x 32 KB ([K;Q] per dk half)
    static constexpr uint32_t P_A = P_KQ + 2 * 32768;
    static constexpr uint32_t P_T = P_A + 64 * kLdT * 4;
    static constexpr uint32_t P_STG = P_T + 64 * kLdT * 4;  // 2 staging slots
    static constexpr uint32_t P_GATE = P_STG + 2 * H_SLOT;  // g[64], beta[64]
    static constexpr uint32_t P_BAR = P_GATE + 512;
    static constexpr uint32_t P_BYTES = P_BAR + 128;
    static constexpr uint32_t kAlloc = (S_BYTES > P_BYTES ? S_BYTES : P_BYTES) + 1024;
};
static_assert(Tc2Layout::S_H % 1024 == 0 && Tc2Layout::S_W % 1024 == 0 && Tc2Layout::S_SB % 1024 == 0,
              "state tiles must be 1024-aligned");
static_assert(Tc2Layout::P_STG % 1024 == 0 && Tc2Layout::H_SLOT % 1024 == 0, "slots must be 1024-aligned");
static_assert(Tc2Layout::kAlloc <= 232448, "shared memory budget");

// state TMEM columns (512 allocated)
constexpr uint32_t kT2S = 0, kT2W = 128, kT2U = 192, kT2O = 320;  // U, O double-buffered (+64)

__device__ __forceinline__ void tc2_gates(int lane, int nv, const float *la, const float *bt, size_t H,
                                          float *g, float *gam, float *beta, float *dec) {
    const int r0 = 2 * lane, r1 = r0 + 1;
    const float l0 = r0 < nv ? la[(size_t)r0 * H] : 0.f;
    const float l1 = r1 < nv ? la[(size_t)r1 * H] : 0.f;
    float incl = l0 + l1;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const float y = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += y;
    }
    const float g1 = incl, g0 = incl - l1;
    const float gC = __shfl_sync(0xffffffffu, incl, 31);
    g[r0] = g0; g[r1] = g1;
    gam[r0] = expf(g0); gam[r1] = expf(g1);
    dec[r0] = expf(gC - g0); dec[r1] = expf(gC - g1);
    beta[r0] = r0 < nv ? bt[(size_t)r0 * H] : 0.f;
    beta[r1] = r1 < nv ? bt[(size_t)r1 * H] : 0.f;
}

// ------------------------------------------------------------------ prep CTA --
__device__ __forceinline__ void tc2_prep(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                         int T, int H, int b, int h, const float *log_alpha,
                                         const float *beta) {
    using L = Tc2Layout;
    using namespace sm100;
    const int tid = threadIdx.x, warp = tid >> 5;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *tma_full = reinterpret_cast<uint64_t *>(sm + L::P_BAR);  // [2]
    uint64_t *empty = tma_full + 2;                                      // [2], arrived by the state CTA
    uint64_t *mma_bar = tma_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *sg = reinterpret_cast<float *>(sm + L::P_GATE), *sbeta = sg + 64;
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
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
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
        const int c0 = n * kChunk, nv = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        uint8_t *stg = sm + L::P_STG + s * L::H_SLOT;
        float *hg = reinterpret_cast<float *>(stg + L::H_G);
        __syncthreads();
        if (*abort_flag) break;
        if (tid == 0) {
            // staging slot s (and the state's slot s) must have been consumed (chunk n-2)
            if (n >= 2 && !mbar_wait_cluster(&empty[s], (uint32_t)(((n >> 1) - 1) & 1))) *abort_flag = 1;
            if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        }
        mma_phase ^= 1;
        if (warp == 0) tc2_gates(tid, nv, log_alpha + tok0, beta + tok0, (size_t)H, sg, hg, sbeta, hg + 64);
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();

        // A (fp32, rows 0-63) and P (bf16 into the staging slot, rows 64-127)
        {
            float v[64];
            tmem_ld32(tl, v);
            tmem_ld32(tl + 32, v + 32);
            if (tid < 64) {
                const int r = tid;
                const float gr = sg[r], br = sbeta[r];
#pragma unroll
                for (int i = 0; i < 64; ++i) sA[r * kLdT + i] = (i < r) ? br * __expf(gr - sg[i]) * v[i] : 0.f;
            } else {
                const int r = tid - 64;
                const float gr = sg[r];
#pragma unroll
                for (int i = 0; i < 64; ++i) v[i] = (i <= r) ? __expf(gr - sg[i]) * v[i] : 0.f;
#pragma unroll
                for (int ch = 0; ch < 8; ++ch) st_bf16x8(stg + L::H_P + sw128_offset(r, ch), v + 8 * ch);
            }
        }
        // Q~ = diag(gamma) Q: same swizzled positions as the Q tile
        {
            const uint8_t *qt = sm + L::P_KQ + s * 32768 + 8192;
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const int ci = tid * 8 + e;  // 16-byte chunk 0..1023
                const int half = ci >> 9;
                const uint32_t ob = (uint32_t)(ci & 511) * 16;
                const float gm = hg[ob >> 7];
                float f[8];
                load8(reinterpret_cast<const __nv_bfloat16 *>(qt + half * 16384 + ob), f);
#pragma unroll
                for (int i = 0; i < 8; ++i) f[i] *= gm;
                st_bf16x8(stg + L::H_QT + half * 8192 + ob, f);
            }
        }
        tc_before_sync();
        __syncthreads();
        if (tid == 0 && n + 1 < nch) {  // next chunk's K K^T / Q K^T overlaps this chunk's solve
            tc_after_sync();
            if (!mbar_wait(&tma_full[s ^ 1], (uint32_t)(((n + 1) >> 1) & 1))) *abort_flag = 1;
            else {
                ++tma_done;
                issue_mma1(s ^ 1);
            }
        }
        invert_unit_lower_64(sA, sT);
        {   // T' = T diag(beta), T'' = T diag(beta gamma)
            const int r = tid & 63;
            const bool second = tid >= 64;
            float v[8];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) {
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int i = ch * 8 + e;
                    const float t = (i <= r) ? sT[r * kLdT + i] : 0.f;
                    v[e] = t * sbeta[i] * (second ? hg[i] : 1.f);
                }
                st_bf16x8(stg + (second ? L::H_T2 : L::H_T1) + sw128_offset(r, ch), v);
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
                                          int T, int H, int b, int h, const float *S0,
                                          __nv_bfloat16 *o, float *S_T) {
    using L = Tc2Layout;
    using namespace sm100;
    constexpr int D = 128;
    const int tid = threadIdx.x, warp = tid >> 5;
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
        mbar_expect_tx(&hand_full[0], L::H_BYTES);  // arm the slots for chunks 0 and 1
        if (nch > 1) mbar_expect_tx(&hand_full[1], L::H_BYTES);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    cluster_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(warp * 32) << 16);
    const uint32_t remote_empty0 = cluster_addr(sm + L::P_BAR + 16, 0);  // prep's empty[0]

    {   // entry state -> TMEM (row tid)
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
            tmem_st32(tl + kT2S + c * 32, v);
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
    auto epilogue = [&](int n) {  // O^T (lane = value channel, column = token) -> o
        const int c0 = n * kChunk, nv = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        float v[32];
#pragma unroll 1
        for (int half = 0; half < 2; ++half) {
            tmem_ld32(tl + kT2O + 64 * (n & 1) + half * 32, v);
#pragma unroll
            for (int i = 0; i < 32; ++i) {
                const int r = half * 32 + i;
                if (r < nv) o[(tok0 + (size_t)r * H) * D + tid] = __float2bfloat16_rn(v[i]);
            }
        }
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
        float v[64];
        tmem_ld32(tl + kT2W, v);
        tmem_ld32(tl + kT2W + 32, v + 32);
#pragma unroll
        for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::S_W + sw128_offset(tid, ch), v + 8 * ch);
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
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                tmem_ld32(tl + kT2S + c * 32, v);
                uint8_t *half = sm + L::S_SB + (c >> 1) * 16384;
#pragma unroll
                for (int q4 = 0; q4 < 4; ++q4) st_bf16x8(half + sw128_offset(tid, (c & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
                for (int i = 0; i < 32; ++i) v[i] *= gC;
                tmem_st32(tl + kT2S + c * 32, v);
            }
            tmem_wait_st();
        }
        fence_async_smem();
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
        // (c) epilogue of the previous chunk, then W/U^g of the next chunk
        if (n > 0) epilogue(n - 1);
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
        {
            float v[64];
            tmem_ld32(tl + kT2U + 64 * s, v);
            tmem_ld32(tl + kT2U + 64 * s + 32, v + 32);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::S_SB + sw128_offset(tid, ch), v + 8 * ch);
#pragma unroll
            for (int i = 0; i < 64; ++i) v[i] *= hgate[64 + i];
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::S_SB + 16384 + sw128_offset(tid, ch), v + 8 * ch);
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
            float v[64];
            tmem_ld32(tl + kT2W, v);
            tmem_ld32(tl + kT2W + 32, v + 32);
#pragma unroll
            for (int ch = 0; ch < 8; ++ch) st_bf16x8(sm + L::S_W + sw128_offset(tid, ch), v + 8 * ch);
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
        epilogue(nch - 1);
        if (S_T) {
            float v[32];
#pragma unroll 1
            for (int c = 0; c < 4; ++c) {
                tmem_ld32(tl + kT2S + c * 32, v);
                float4 *dst = reinterpret_cast<float4 *>(S_T + ((size_t)bh * D + tid) * D + c * 32);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
        }
    }
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        // drain: this CTA's TMA loads, its MMAs, and the prep CTA's copies into it
        for (int k2 = tma_done_n; k2 < tma_issued; ++k2) mbar_wait(&tma_full[k2 & 1], (uint32_t)((k2 >> 1) & 1));
        mma_commit(bar_a);
        mbar_wait(bar_a, aphase);
        for (int k2 = n_done; k2 < nch && k2 < n_done + 2; ++k2)
            mbar_wait_cluster(&hand_full[k2 & 1], (uint32_t)((k2 >> 1) & 1));
    }
    (void)n_done;
    tc_before_sync();
    __syncthreads();
    cluster_sync();
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTcThreads, 1)
gdr_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, int T, int H,
                   const float *__restrict__ log_alpha, const float *__restrict__ beta,
                   const float *__restrict__ S0, __nv_bfloat16 *__restrict__ o, float *__restrict__ S_T) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int bh = blockIdx.x >> 1, b = bh / H, h = bh % H;
    if (sm100::cluster_ctarank() == 0)
        tc2_prep(sm, &tm_q, &tm_k, T, H, b, h, log_alpha, beta);
    else
        tc2_state(sm, &tm_k, &tm_v, T, H, b, h, S0, o, S_T);
}

inline cudaError_t launch_fwd_tc2(int B, int T, int H, const void *q, const void *k, const void *v,
                                  const float *la, const float *beta, const float *S0, void *o,
                                  float *S_T, cudaStream_t stream) {
    CUtensorMap mq, mk, mv;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr_fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)Tc2Layout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr_fwd_tc2_kernel<<<(unsigned)(2 * B * H), kTcThreads, Tc2Layout::kAlloc, stream>>>(
        mq, mk, mv, T, H, la, beta, S0, static_cast<__nv_bfloat16 *>(o), S_T);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
