// bwd_tc.cuh -- chunkwise backward of the gated delta rule on the tensor cores
// (bf16 q/k/v/dO, dk = dv = 128, fp32 state and gradients of the state).
//
// The pages give no backward; the reverse mode here is the chain rule applied
// to the chunk map of the forward (chunkwise form of the Gated DeltaNet
// review, meaningful96.github.io/nr/GDN, section 3.7; the per-chunk formulas
// are listed at the top of bwd_simt.cuh).  Three steps in two launches (1
// and 2 share one launch, gdr_bwd_passes_kernel, as they are independent):
//
//  1. the forward, recomputed without outputs, keeps every chunk's entry
//     state S_n as its bf16 MMA operand tile (32 KB, 128B-swizzled);
//  2. the dS pass, one 2-CTA cluster per (b, h), walks
//     the chunks from last to first.  Its prep CTA is the forward's (masks,
//     inverse, P, Q~ = diag(gamma) Q, T'' = T diag(beta gamma)); its state CTA
//     carries D = dL/dS (exit state of the current chunk) in TMEM:
//        dU^T = D K^T diag(exp(g_C - g)) + dO^T P
//        D   <- gamma_C D + dO^T Q~ - dU^T W,   W = T'' K,
//     and stores every chunk's D the same way for step 3;  dS0 is the final
//     D (fp32);
//  3. the gradients (gdr_bwd_grad_kernel), one CTA per (b, h, chunk), all
//     chunks in parallel, from S_n, D_n and the chunk's inputs.
#pragma once
#include "fwd_tc2.cuh"

namespace gdr {

// TMEM columns of the dS pass (512 allocated)
constexpr uint32_t kBcD = 0, kBcX1 = 128, kBcX2 = 192, kBcW = 256;

// State CTA of the dS pass.  Shared memory follows Tc2Layout (the prep CTA's
// DSMEM copies land in S_H): K tiles in S_K, dO tiles in S_V, W in S_W, bf16
// D and then dU^T in S_SB.  W of step n+1 is computed behind step n's D
// update and converted in step n+1, so the hand-off wait stays off the chain.
__device__ __forceinline__ void bwd_chain_state(uint8_t *sm, const CUtensorMap *tm_k, const CUtensorMap *tm_do,
                                                int T, int H, int b, int h, const float *dS_T, float *dS0,
                                                uint8_t *D_tiles) {
    using L = Tc2Layout;
    using namespace sm100;
    constexpr int D = 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;           // TMEM lane = row of D / dU^T / W^T
    const int bh = b * H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *tma_full = reinterpret_cast<uint64_t *>(sm + L::S_BAR);  // [2]
    uint64_t *hand_full = tma_full + 2;                                  // [2], filled by the prep CTA
    uint64_t *bar_a = tma_full + 4, *bar_b = tma_full + 5;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_full + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t sbase = smem_u32(sm);
    auto chunk_of = [&](int n) { return nch - 1 - n; };

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
        prefetch_tmap(tm_do);
        mbar_expect_tx(&hand_full[0], L::H_BYTES);  // arm the slots for steps 0 and 1
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

    {   // seed D = dS_T (or 0) -> TMEM
        float v[32];
        const int col = wc * 32;
        if (dS_T) {
            const float4 *src = reinterpret_cast<const float4 *>(dS_T + ((size_t)bh * D + row) * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 x = src[i];
                v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        tmem_st32(tl + kBcD + col, v);
        tmem_wait_st();
    }

    auto issue_tma = [&](int n, int s) {
        uint8_t *kt = sm + L::S_K + s * 16384, *dt = sm + L::S_V + s * 16384;
        const int c = chunk_of(n);
        mbar_expect_tx(&tma_full[s], 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(kt + half * 8192, tm_k, &tma_full[s], half * 64, h, c * kChunk, b);
            tma_load_4d(dt + half * 8192, tm_do, &tma_full[s], half * 64, h, c * kChunk, b);
        }
    };
    // W^T = K^T T''^T of step n (thread 0), after its inputs landed
    auto issue_w = [&](int n) -> bool {
        const int s = n & 1;
        if (!mbar_wait(&tma_full[s], (uint32_t)((n >> 1) & 1))) return false;
        if (!mbar_wait_cluster(&hand_full[s], (uint32_t)((n >> 1) & 1))) return false;
        tc_after_sync();
        const uint32_t kt = sbase + L::S_K + s * 16384, hs = sbase + L::S_H + s * L::H_SLOT;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kBcW, smem_desc_sw128(kt + kk * 2048, 8192, 1024),
                     smem_desc_sw128(hs + L::H_T2 + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
        mma_commit(bar_b);
        return true;
    };
    auto convert_w = [&]() {  // W^T (lane j, column r) -> [j][r] bf16, the K-major B of D -= dU^T W
        float v[16];
        tmem_ld16(tl + kBcW + wc * 16, v);
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::S_W + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
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
        if (!issue_w(0)) *abort_flag = 1;
        else tma_done_n = 1;
    }
    __syncthreads();

    int n_done = 0;  // steps whose MMAs all completed
#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        if (*abort_flag) break;
        const int s = n & 1, c = chunk_of(n);
        const uint32_t hs = sbase + L::S_H + s * L::H_SLOT;
        const float *hgate = reinterpret_cast<const float *>(sm + L::S_H + s * L::H_SLOT + L::H_G);

        // (a) D (the exit-state gradient of chunk c) -> bf16 operand; D *= gamma_C
        {
            const float gC = hgate[kChunk - 1];
            const int col = wc * 32;
            float v[32];
            tmem_ld32(tl + kBcD + col, v);
            uint8_t *half = sm + L::S_SB + (wc >> 1) * 16384;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) st_bf16x8(half + sw128_offset(row, (wc & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= gC;
            tmem_st32(tl + kBcD + col, v);
            tmem_wait_st();
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // (b) X1 = D K^T, X2 = dO^T P (-> bar_a); then D += dO^T Q~
        if (tid == 0) {
            tc_after_sync();
            if (D_tiles) {  // the bf16 tile of D, as swizzled, for the gradient kernel
                bulk_store_s2g(D_tiles + ((size_t)bh * nch + c) * 32768, sm + L::S_SB, 32768);
                bulk_commit();
            }
            const uint32_t sb = sbase + L::S_SB;
            const uint32_t kt = sbase + L::S_K + s * 16384, dt = sbase + L::S_V + s * 16384;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kBcX1, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(kt + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBcX2, smem_desc_sw128(dt + kk * 2048, 8192, 1024),
                         smem_desc_sw128(hs + L::H_P + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true),
                         kk > 0);
            mma_commit(bar_a);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBcD, smem_desc_sw128(dt + kk * 2048, 8192, 1024),
                         smem_desc_sw128(hs + L::H_QT + kk * 2048, 8192, 1024), idesc_bf16(128, 128, true, true), 1);
        }
        __syncwarp();
        // (d) dU^T = X1 diag(exp(g_C - g)) + X2 -> bf16 A operand; W of this step -> S_W
        if (tid == 0) {
            if (!mbar_wait(bar_a, aphase) || !mbar_wait(bar_b, bphase)) *abort_flag = 1;
            if (D_tiles) bulk_wait_read_all();  // the copy of D has left S_SB
        }
        aphase ^= 1;
        bphase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        {
            float x1[16], x2[16];
            tmem_ld16x2(tl + kBcX1 + wc * 16, x1, tl + kBcX2 + wc * 16, x2);
#pragma unroll
            for (int k4 = 0; k4 < 4; ++k4) {
                const float4 dv4 = *reinterpret_cast<const float4 *>(hgate + 64 + wc * 16 + 4 * k4);
                x1[4 * k4] = fmaf(x1[4 * k4], dv4.x, x2[4 * k4]);
                x1[4 * k4 + 1] = fmaf(x1[4 * k4 + 1], dv4.y, x2[4 * k4 + 1]);
                x1[4 * k4 + 2] = fmaf(x1[4 * k4 + 2], dv4.z, x2[4 * k4 + 2]);
                x1[4 * k4 + 3] = fmaf(x1[4 * k4 + 3], dv4.w, x2[4 * k4 + 3]);
            }
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::S_SB + sw128_offset(row, wc * 2 + ch), x1 + 8 * ch);
        }
        convert_w();
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // (e) D -= dU^T W, then W of the next step
        if (tid == 0) {
            tc_after_sync();
            const uint32_t du = sbase + L::S_SB, wb = sbase + L::S_W;
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBcD, smem_desc_sw128(du + kk * 32, 16, 1024), smem_desc_sw128(wb + kk * 32, 16, 1024),
                         idesc_bf16(128, 128, false, false, true), 1);
            mma_commit(bar_a);
            if (n + 1 < nch) {
                if (!issue_w(n + 1)) *abort_flag = 1;
                else ++tma_done_n;
            }
        }
        // (g) step n finished: release its hand-off slot and K/dO stage
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

    if (!*abort_flag && dS0) {
        float v[32];
        const int col = wc * 32;
        tmem_ld32(tl + kBcD + col, v);
        float4 *dst = reinterpret_cast<float4 *>(dS0 + ((size_t)bh * D + row) * D + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    if (tid == 0) bulk_wait_all();  // the copies of D are complete before the CTA exits
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

// The recompute and the dS pass need nothing from each other, so one launch
// runs both: clusters [0, B*H) recompute the forward (no outputs, bf16 state
// tiles kept), clusters [B*H, 2*B*H) run the dS pass.
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kTc2Threads, 1)
gdr_bwd_passes_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                      const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                      int T, int H, const float *__restrict__ log_alpha, const float *__restrict__ beta,
                      const float *__restrict__ S0, const float *__restrict__ dS_T, float *__restrict__ dS0,
                      uint8_t *__restrict__ S_tiles, uint8_t *__restrict__ D_tiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int nbh = (int)(gridDim.x >> 2), cl = (int)(blockIdx.x >> 1);
    const bool dS_pass = cl >= nbh;
    const int bh = dS_pass ? cl - nbh : cl, b = bh / H, h = bh % H;
    if (sm100::cluster_ctarank() == 0)
        tc2_prep(sm, &tm_q, &tm_k, T, H, b, h, log_alpha, beta, dS_pass);
    else if (dS_pass)
        bwd_chain_state(sm, &tm_k, &tm_do, T, H, b, h, dS_T, dS0, D_tiles);
    else  // no output: the q map stands in for the unused output map
        tc2_state(sm, &tm_k, &tm_v, &tm_q, T, H, b, h, S0, nullptr, false, S_tiles);
}

// ------------------------------------------------------------ gradient kernel --
// One CTA per (b, h, chunk); with S = S_n, D = D_n (fp32 from the two passes
// above), C = 64, d = 128, and every product laid out with d on the MMA's M
// (TMEM lane = c or j, column = token r or i):
//   G1  [K K^T; Q K^T]          X^T|Y^T = S [K; Q]^T     X1 = D K^T       dQ1^T = S^T dO^T
//   G2  U^T = R^T T^T, R = diag(beta)(V - diag(gamma) X)                 X2 = dO^T P
//   G3  dR^T = dU^T T, dU^T = X1 diag(exp(g_C - g)) + X2                 (U D)^T = D^T U^T
//   G4  [dA'; dP] = [dR; dO] U^T  (dA = -dA')                            (dR S)^T = S^T dR^T
//   G5  dQ2^T = K^T (dP*L)^T      dK12^T = Q^T (dP*L) + K^T (dKK + dKK^T), dKK = dA * beta_r Gamma
// and then dq = diag(gamma) dQ1 + dQ2, dk = dK12 + diag(exp(g_C - g)) U D - diag(beta gamma) dR S,
// dv = diag(beta) dR, dbeta and dg by the row/column sums of the formulas in
// bwd_simt.cuh, dlog alpha as the in-chunk suffix sums of dg.
struct BgLayout {
    static constexpr uint32_t KQ = 0;          // [K; Q] per dk half: K rows at +0, Q rows at +8192
    static constexpr uint32_t V = 32768;       // V, 2 halves x 8 KB
    static constexpr uint32_t DOR = 49152;     // [dR; dO] per dv half: dR rows at +0, dO rows at +8192
    static constexpr uint32_t SB = 81920;      // S bf16 [c][j], 2 halves x 16 KB
    static constexpr uint32_t DB = 114688;     // D bf16 [c][j]
    static constexpr uint32_t RU = 147456;     // R^T, then dU^T, [c][r] bf16
    static constexpr uint32_t UB = 163840;     // U^T [c][r] bf16
    static constexpr uint32_t TB = 180224;     // T bf16 [r][i], then dKK + dKK^T
    static constexpr uint32_t FT = UB;         // T fp32 (64 x kLdT), overlaps UB and the first 1 KB of TB
    static constexpr uint32_t PB = 188416;     // P bf16 [r][i], then dP * L
    static constexpr uint32_t FA = 196608;     // A fp32 (64 x kLdT), then dKK
    static constexpr uint32_t GATE = FA + 64 * kLdT * 4;  // g, beta, gamma, dec [64] each
    static constexpr uint32_t RED = GATE + 1024;          // fixed-order partial sums (floats):
    static constexpr uint32_t R6DB = 0, R6DG = 256;       //   [4 lane quarters][64]
    static constexpr uint32_t R8RDB = 512;                //   [4 column groups][64]
    static constexpr uint32_t R8RDG = 768;                //   [4 column groups][128]
    static constexpr uint32_t R8C = 1280;                 //   [4 lane quarters][64]
    static constexpr uint32_t RDS = 1536, RDGC = 1552;    //   [16 warps] each
    static constexpr uint32_t BAR = RED + 1568 * 4;
    static constexpr uint32_t BYTES = BAR + 64;
    static constexpr uint32_t kAlloc = BYTES + 1024;
};
static_assert(BgLayout::FT + 64 * kLdT * 4 <= BgLayout::TB + 1024, "T scratch overlaps one row group of TB");
static_assert(BgLayout::GATE % 16 == 0 && BgLayout::BAR % 8 == 0, "alignment");
static_assert(BgLayout::kAlloc <= 232448, "shared memory budget");

// TMEM columns of the gradient kernel (512 allocated)
constexpr uint32_t kBgKQ = 0, kBgX = 64, kBgY = 128, kBgX1 = 192, kBgDQ1 = 256, kBgU = 320, kBgX2 = 384;
constexpr uint32_t kBgDR = 192, kBgUD = 384, kBgPA = 448, kBgDRS = 64, kBgDQ2 = 128, kBgDK = 192;

// Sums v[0..15] over the 32 lanes of a warp in a fixed order: afterwards lane
// l holds the sum for index l & 15 (lanes l and l + 16 agree).
__device__ __forceinline__ float warp_sum16_transposed(float (&v)[16], int lane) {
    float w[8];
    {
        const bool hi = (lane & 8) != 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float send = hi ? v[i] : v[i + 8];
            const float keep = hi ? v[i + 8] : v[i];
            w[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
        }
    }
    float x[4];
    {
        const bool hi = (lane & 4) != 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const float send = hi ? w[i] : w[i + 4];
            const float keep = hi ? w[i + 4] : w[i];
            x[i] = keep + __shfl_xor_sync(0xffffffffu, send, 4);
        }
    }
    float y[2];
    {
        const bool hi = (lane & 2) != 0;
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const float send = hi ? x[i] : x[i + 2];
            const float keep = hi ? x[i + 2] : x[i];
            y[i] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
        }
    }
    const bool hi = (lane & 1) != 0;
    float z = (hi ? y[1] : y[0]) + __shfl_xor_sync(0xffffffffu, hi ? y[0] : y[1], 1);
    return z + __shfl_xor_sync(0xffffffffu, z, 16);
}

__device__ __forceinline__ float warp_sum32(float x) {
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

__global__ void __launch_bounds__(kTc2Threads, 1)
gdr_bwd_grad_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_do,
                    int T, int H, const float *__restrict__ log_alpha, const float *__restrict__ beta,
                    const uint8_t *__restrict__ S_tiles, const uint8_t *__restrict__ D_tiles,
                    const __grid_constant__ CUtensorMap tm_dq, const __grid_constant__ CUtensorMap tm_dk,
                    const __grid_constant__ CUtensorMap tm_dv, float *__restrict__ dlog_alpha,
                    float *__restrict__ dbeta) {
    using L = BgLayout;
    using namespace sm100;
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;           // TMEM lane
    const int nch = (T + kChunk - 1) / kChunk;
    const int c = blockIdx.x % nch, bh = blockIdx.x / nch, b = bh / H, h = bh % H;
    const int t0 = c * kChunk, nv = min(kChunk, T - t0);
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR), *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *sg = reinterpret_cast<float *>(sm + L::GATE), *sbeta = sg + 64, *sgam = sg + 128, *sdec = sg + 192;
    float *red = reinterpret_cast<float *>(sm + L::RED);
    float *sA = reinterpret_cast<float *>(sm + L::FA), *sT = reinterpret_cast<float *>(sm + L::FT);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t kq = sbase + L::KQ, dor = sbase + L::DOR, sb = sbase + L::SB, db = sbase + L::DB;
    const uint32_t ru = sbase + L::RU, ub = sbase + L::UB, tb = sbase + L::TB, pb = sbase + L::PB;
    const size_t chunk_tile = ((size_t)bh * nch + c) * 32768;
    auto tok = [&](int r) { return ((size_t)(b * T + t0 + r) * H + h); };

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *abort_flag = 0;
        mbar_expect_tx(bar_tma, 65536 + 2 * 32768);
        bulk_load_g2s(sm + L::SB, S_tiles + chunk_tile, 32768, bar_tma);
        bulk_load_g2s(sm + L::DB, D_tiles + chunk_tile, 32768, bar_tma);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(sm + L::KQ + half * 16384, &tm_k, bar_tma, half * 64, h, t0, b);
            tma_load_4d(sm + L::KQ + half * 16384 + 8192, &tm_q, bar_tma, half * 64, h, t0, b);
            tma_load_4d(sm + L::V + half * 8192, &tm_v, bar_tma, half * 64, h, t0, b);
            tma_load_4d(sm + L::DOR + half * 16384 + 8192, &tm_do, bar_tma, half * 64, h, t0, b);
        }
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    if (warp == 15) {  // gates: g (inclusive prefix sum of log alpha), beta, gamma, exp(g_C - g)
        const int r0 = 2 * lane, r1 = r0 + 1;
        const float l0 = r0 < nv ? log_alpha[tok(r0)] : 0.f, l1 = r1 < nv ? log_alpha[tok(r1)] : 0.f;
        const float b0 = r0 < nv ? beta[tok(r0)] : 0.f, b1 = r1 < nv ? beta[tok(r1)] : 0.f;
        float incl = l0 + l1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const float g1 = incl, g0 = incl - l1, gC = __shfl_sync(0xffffffffu, incl, 31);
        sg[r0] = g0; sg[r1] = g1;
        sbeta[r0] = b0; sbeta[r1] = b1;
        sgam[r0] = expf(g0); sgam[r1] = expf(g1);
        sdec[r0] = expf(gC - g0); sdec[r1] = expf(gC - g1);
    }
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    uint32_t mph = 0;
    int ncommit = 0;  // commits of bar_mma issued by thread 0
    bool tma_pending = true;
    // every thread: wait for the last commit of bar_mma
    auto mma_wait_all = [&]() -> bool {
        if (tid == 0 && !*abort_flag && !mbar_wait(bar_mma, mph)) *abort_flag = 1;
        mph ^= 1;
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
        return *abort_flag == 0;
    };
    // publish shared-memory operands to the tensor cores
    auto operands_ready = [&]() {
        fence_async_smem();
        tc_before_sync();
        __syncthreads();
    };

    do {
        // ---- G1
        if (tid == 0) {
            if (!mbar_wait(bar_tma, 0)) *abort_flag = 1;
            else {
                tma_pending = false;
                tc_after_sync();
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    const uint64_t a = smem_desc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024);
                    mma_bf16(tmem + kBgKQ, a, a, idesc_bf16(128, 64, false, false), kk > 0);
                }
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + kBgX, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             smem_desc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             idesc_bf16(128, 128, false, false), kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + kBgX1, smem_desc_sw128(db + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             smem_desc_sw128(kq + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk)
                    mma_bf16(tmem + kBgDQ1, smem_desc_sw128(sb + kk * 2048, 16384, 1024),
                             smem_desc_sw128(dor + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                             idesc_bf16(128, 64, true, false), kk > 0);
                mma_commit(bar_mma);
                ++ncommit;
            }
        }
        if (!mma_wait_all()) break;

        {   // <D, S> over the bf16 tiles (same layout, so elementwise by byte offset)
            float ds = 0.f;
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                float fs[8], fd[8];
                const uint32_t off = (uint32_t)(tid + m * kTc2Threads) * 16;
                load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::SB + off), fs);
                load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::DB + off), fd);
#pragma unroll
                for (int i = 0; i < 8; ++i) ds = fmaf(fs[i], fd[i], ds);
            }
            ds = warp_sum32(ds);
            if (lane == 0) red[L::RDS + warp] = ds;
        }
        // ---- masks: A (fp32, rows 0-63) and P (bf16, rows 64-127); R^T from X^T
        {
            float v[16];
            tmem_ld16(tl + kBgKQ + wc * 16, v);
            const int i0 = wc * 16;
            if (row < 64) {
                const int r = row;
                const float gr = sg[r], br = sbeta[r];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = (i0 + i < r) ? br * __expf(gr - sg[i0 + i]) * v[i] : 0.f;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    *reinterpret_cast<float4 *>(sA + r * kLdT + i0 + 4 * k4) =
                        make_float4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
            } else {
                const int r = row - 64;
                const float gr = sg[r];
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = (i0 + i <= r) ? __expf(gr - sg[i0 + i]) * v[i] : 0.f;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::PB + sw128_offset(r, wc * 2 + ch), v + 8 * ch);
            }
        }
        {
            float x[16];
            tmem_ld16(tl + kBgX + wc * 16, x);
            const int cc = row;
            const uint8_t *vh = sm + L::V + (cc >> 6) * 8192;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = wc * 16 + i;
                x[i] = sbeta[r] * (ld_sw_bf16(vh, r, cc & 63) - sgam[r] * x[i]);
            }
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::RU + sw128_offset(cc, wc * 2 + ch), x + 8 * ch);
        }
        __syncthreads();
        if (warp < 2) inverse_two_warps(sA, sT, warp, lane, 1, TEmit{nullptr, nullptr, nullptr, nullptr});
        __syncthreads();
        {   // T fp32 -> bf16 [r][i] (lower triangle; the fp32 scratch overlaps TB)
            const int r = tid & 63, cb = (tid >> 6) * 8;
            float t[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) t[q] = (cb + q <= r) ? sT[r * kLdT + cb + q] : 0.f;
            __syncthreads();
            st_bf16x8(sm + L::TB + sw128_offset(r, cb >> 3), t);
        }
        operands_ready();

        // ---- G2: U^T = R^T T^T, X2 = dO^T P
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBgU, smem_desc_sw128(ru + kk * 32, 16, 1024), smem_desc_sw128(tb + kk * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBgX2, smem_desc_sw128(dor + 8192 + kk * 2048, 16384, 1024),
                         smem_desc_sw128(pb + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;
        {   // U^T -> bf16; dU^T = X1 diag(exp(g_C - g)) + X2 -> bf16 (over R^T)
            float u[16];
            tmem_ld16(tl + kBgU + wc * 16, u);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::UB + sw128_offset(row, wc * 2 + ch), u + 8 * ch);
            float x1[16], x2[16];
            tmem_ld16x2(tl + kBgX1 + wc * 16, x1, tl + kBgX2 + wc * 16, x2);
#pragma unroll
            for (int i = 0; i < 16; ++i) x1[i] = fmaf(x1[i], sdec[wc * 16 + i], x2[i]);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::RU + sw128_offset(row, wc * 2 + ch), x1 + 8 * ch);
        }
        operands_ready();

        // ---- G3: dR^T = dU^T T, (U D)^T = D^T U^T
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBgDR, smem_desc_sw128(ru + kk * 32, 16, 1024),
                         smem_desc_sw128(tb + kk * 2048, 8192, 1024), idesc_bf16(128, 64, false, true), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kBgUD, smem_desc_sw128(db + kk * 2048, 16384, 1024),
                         smem_desc_sw128(ub + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;

        // ---- dR (bf16, K-major rows r, for G4), dv, and the d-reductions of dbeta and dg
        {
            const int cc = row;  // value channel c for dR^T / X^T / Y^T, key channel j for (U D)^T
            float rb[16], rg[16], rc = 0.f;
            {
                float dr[16], x[16];
                tmem_ld16x2(tl + kBgDR + wc * 16, dr, tl + kBgX + wc * 16, x);
                uint8_t *drh = sm + L::DOR + (cc >> 6) * 16384, *dvh = sm + L::DB + (cc >> 6) * 8192;
                const uint8_t *vh = sm + L::V + (cc >> 6) * 8192;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = wc * 16 + i;
                    const float gr = sgam[r], br = sbeta[r];
                    rb[i] = dr[i] * (ld_sw_bf16(vh, r, cc & 63) - gr * x[i]);
                    rg[i] = -br * gr * dr[i] * x[i];
                    st_sw_bf16(drh, r, cc & 63, dr[i]);
                    st_sw_bf16(dvh, r, cc & 63, br * dr[i]);  // dv tile (D is dead by now)
                }
            }
            {
                float y[16];
                tmem_ld16(tl + kBgY + wc * 16, y);
                const uint8_t *doh = sm + L::DOR + (cc >> 6) * 16384 + 8192;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = wc * 16 + i;
                    rg[i] = fmaf(sgam[r] * ld_sw_bf16(doh, r, cc & 63), y[i], rg[i]);
                }
            }
            {
                float ud[16];
                tmem_ld16(tl + kBgUD + wc * 16, ud);
                const uint8_t *kh = sm + L::KQ + (cc >> 6) * 16384;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const int r = wc * 16 + i;
                    const float t = sdec[r] * ud[i] * ld_sw_bf16(kh, r, cc & 63);
                    rg[i] -= t;
                    rc += t;
                }
            }
            const float sb16 = warp_sum16_transposed(rb, lane);
            const float sg16 = warp_sum16_transposed(rg, lane);
            rc = warp_sum32(rc);
            if (lane < 16) {
                red[L::R6DB + wq * 64 + wc * 16 + lane] = sb16;
                red[L::R6DG + wq * 64 + wc * 16 + lane] = sg16;
            }
            if (lane == 0) red[L::RDGC + warp] = rc;
        }
        operands_ready();

        // ---- G4: [dA'; dP] = [dR; dO] U^T, (dR S)^T = S^T dR^T
        if (tid == 0) {
            tma_store_4d(&tm_dv, sm + L::DB, 0, h, t0, b);  // dv [token][channel], tokens past T clipped
            tma_store_4d(&tm_dv, sm + L::DB + 8192, 64, h, t0, b);
            bulk_commit();
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kBgPA, smem_desc_sw128(dor + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(ub + kk * 2048, 8192, 1024), idesc_bf16(128, 64, false, true), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kBgDRS, smem_desc_sw128(sb + kk * 2048, 16384, 1024),
                         smem_desc_sw128(dor + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, true, false), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;
        {   // rows 0-63: dA, dKK (fp32 -> FA); rows 64-127: dP, dP*L (bf16 -> PB); row and column sums
            float pa[16], kv[16], cs[16];
            tmem_ld16x2(tl + kBgPA + wc * 16, pa, tl + kBgKQ + wc * 16, kv);
            const int i0 = wc * 16;
            float rs_b = 0.f, rs_g = 0.f;
            if (row < 64) {
                const int r = row;
                const float gr = sg[r], br = sbeta[r];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (i0 + i < r) {
                        const float gm = __expf(gr - sg[i0 + i]);
                        const float G = gm * kv[i], dA = -pa[i];
                        rs_b = fmaf(dA, G, rs_b);
                        cs[i] = dA * br * G;
                        rs_g += cs[i];
                        pa[i] = dA * br * gm;
                    } else {
                        cs[i] = 0.f;
                        pa[i] = 0.f;
                    }
                }
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    *reinterpret_cast<float4 *>(sA + r * kLdT + i0 + 4 * k4) =
                        make_float4(pa[4 * k4], pa[4 * k4 + 1], pa[4 * k4 + 2], pa[4 * k4 + 3]);
                red[L::R8RDB + wc * 64 + r] = rs_b;
            } else {
                const int r = row - 64;
                const float gr = sg[r];
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    if (i0 + i <= r) {
                        const float lm = __expf(gr - sg[i0 + i]);
                        cs[i] = pa[i] * lm * kv[i];
                        rs_g += cs[i];
                        pa[i] *= lm;
                    } else {
                        cs[i] = 0.f;
                        pa[i] = 0.f;
                    }
                }
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::PB + sw128_offset(r, wc * 2 + ch), pa + 8 * ch);
            }
            red[L::R8RDG + wc * 128 + row] = rs_g;
            const float col = warp_sum16_transposed(cs, lane);
            if (lane < 16) red[L::R8C + wq * 64 + i0 + lane] = col;
        }
        __syncthreads();
        {   // dKK + dKK^T -> bf16 [r][i] (over T)
            const int r = tid & 63, cb = (tid >> 6) * 8;
            float m[8];
#pragma unroll
            for (int q = 0; q < 8; ++q) m[q] = sA[r * kLdT + cb + q] + sA[(cb + q) * kLdT + r];
            st_bf16x8(sm + L::TB + sw128_offset(r, cb >> 3), m);
        }
        operands_ready();

        // ---- G5: dQ2^T = K^T (dP*L)^T;  dK12^T = Q^T (dP*L) + K^T (dKK + dKK^T)
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBgDQ2, smem_desc_sw128(kq + kk * 2048, 16384, 1024),
                         smem_desc_sw128(pb + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBgDK, smem_desc_sw128(kq + 8192 + kk * 2048, 16384, 1024),
                         smem_desc_sw128(pb + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kBgDK, smem_desc_sw128(kq + kk * 2048, 16384, 1024),
                         smem_desc_sw128(tb + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), 1);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;

        // ---- dq, dk (lane = key channel j, column = token r)
        {
            const int j = row;
            float a[16], e[16];
            tmem_ld16x2(tl + kBgDQ1 + wc * 16, a, tl + kBgDQ2 + wc * 16, e);
            uint8_t *tq = sm + L::SB + (j >> 6) * 8192, *tk = sm + L::SB + 16384 + (j >> 6) * 8192;  // S is dead
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = wc * 16 + i;
                st_sw_bf16(tq, r, j & 63, fmaf(sgam[r], a[i], e[i]));
            }
            tmem_ld16x2(tl + kBgDK + wc * 16, a, tl + kBgUD + wc * 16, e);
#pragma unroll
            for (int i = 0; i < 16; ++i) a[i] = fmaf(sdec[wc * 16 + i], e[i], a[i]);
            tmem_ld16(tl + kBgDRS + wc * 16, e);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = wc * 16 + i;
                st_sw_bf16(tk, r, j & 63, a[i] - sbeta[r] * sgam[r] * e[i]);
            }
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0) {
            tma_store_4d(&tm_dq, sm + L::SB, 0, h, t0, b);
            tma_store_4d(&tm_dq, sm + L::SB + 8192, 64, h, t0, b);
            tma_store_4d(&tm_dk, sm + L::SB + 16384, 0, h, t0, b);
            tma_store_4d(&tm_dk, sm + L::SB + 16384 + 8192, 64, h, t0, b);
            bulk_commit();
        }
        // ---- dbeta, dg -> dlog alpha (suffix sums inside the chunk)
        if (warp == 0) {
            float dgv[2], dbv[2];
#pragma unroll
            for (int u = 0; u < 2; ++u) {
                const int r = 2 * lane + u;
                float g = 0.f, bb = 0.f;
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    g += red[L::R6DG + q * 64 + r] + red[L::R8RDG + q * 128 + r] +
                         red[L::R8RDG + q * 128 + 64 + r] - red[L::R8C + q * 64 + r];
                    bb += red[L::R6DB + q * 64 + r] + red[L::R8RDB + q * 64 + r];
                }
                if (r == kChunk - 1) {  // g_C: gamma_C <D, S> + sum_r exp(g_C - g_r) (U D)_r . K_r
                    float ds = 0.f, gc = 0.f;
                    for (int w = 0; w < 16; ++w) {
                        ds += red[L::RDS + w];
                        gc += red[L::RDGC + w];
                    }
                    g += sgam[kChunk - 1] * ds + gc;
                }
                dgv[u] = g;
                dbv[u] = bb;
            }
            const float tot = dgv[0] + dgv[1];
            float incl = tot;  // sum over lanes >= this one
#pragma unroll
            for (int off = 1; off < 32; off <<= 1) {
                const float y = __shfl_down_sync(0xffffffffu, incl, off);
                if (lane + off < 32) incl += y;
            }
            const float excl = incl - tot;
            const int r0 = 2 * lane, r1 = r0 + 1;
            if (r0 < nv) {
                dlog_alpha[tok(r0)] = incl;
                dbeta[tok(r0)] = dbv[0];
            }
            if (r1 < nv) {
                dlog_alpha[tok(r1)] = dgv[1] + excl;
                dbeta[tok(r1)] = dbv[1];
            }
        }
    } while (0);

    if (tid == 0) bulk_wait_all();  // the gradient tiles have left shared memory
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        if (tma_pending) mbar_wait(bar_tma, 0);
        mma_commit(bar_mma);  // completes phase ncommit once every MMA issued so far is done
        mbar_wait(bar_mma, (uint32_t)(ncommit & 1));
    }
    tc_before_sync();
    __syncthreads();
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 512);
    }
}

// Workspace of the tensor-core backward: the tiles of S_n, then those of D_n,
// [B, H, nchunks] x 32 KB each.
inline size_t bwd_tc_state_bytes(int B, int T, int H) {
    const size_t nch = (size_t)(T + kChunk - 1) / kChunk;
    return ((size_t)B * H * nch * 32768 + 255) / 256 * 256;
}

inline cudaError_t launch_bwd_tc(int B, int T, int H, const void *q, const void *k, const void *v,
                                 const float *la, const float *beta, const float *S0, const void *dO,
                                 const float *dS_T, void *dq, void *dk_out, void *dv_out, float *dla,
                                 float *dbeta, float *dS0, void *ws, cudaStream_t stream) {
    uint8_t *states = static_cast<uint8_t *>(ws);
    uint8_t *dchunks = states + bwd_tc_state_bytes(B, T, H);
    CUtensorMap mq, mk, mv, mdo;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128) || !make_token_map(&mdo, dO, B, T, H, 128))
        return cudaErrorInvalidValue;
    // 1+2) forward recompute (every chunk's entry state) and dS pass, one launch
    cudaError_t err = cudaFuncSetAttribute(gdr_bwd_passes_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)Tc2Layout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr_bwd_passes_kernel<<<(unsigned)(4 * B * H), kTc2Threads, Tc2Layout::kAlloc, stream>>>(
        mq, mk, mv, mdo, T, H, la, beta, S0, dS_T, dS0, states, dchunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    // 3) all chunks' gradients in parallel
    err = cudaFuncSetAttribute(gdr_bwd_grad_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)BgLayout::kAlloc);
    if (err != cudaSuccess) return err;
    const int nch = (T + kChunk - 1) / kChunk;
    CUtensorMap mdq, mdk, mdv;
    if (!make_token_map(&mdq, dq, B, T, H, 128) || !make_token_map(&mdk, dk_out, B, T, H, 128) ||
        !make_token_map(&mdv, dv_out, B, T, H, 128))
        return cudaErrorInvalidValue;
    gdr_bwd_grad_kernel<<<(unsigned)(B * H * nch), kTc2Threads, BgLayout::kAlloc, stream>>>(
        mq, mk, mv, mdo, T, H, la, beta, states, dchunks, mdq, mdk, mdv, dla, dbeta);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
