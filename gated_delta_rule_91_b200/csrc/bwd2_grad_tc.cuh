// bwd2_grad_tc.cuh -- the Gated DeltaNet-2 backward's per-chunk work on
// tcgen05, one CTA per (b, h, chunk) (bf16 with dk = dv = 128): from every
// chunk's entry state S and exit-state gradient D (the recompute and the dS
// pass, bwd2_ds.cuh) and the chunk's T = (I + A)^{-1} and P, all gradients
// of the chunk's tokens.
//
// The chunk form of the reverse (bwd2_simt.cuh header; Gated DeltaNet-2,
// agihunt.info/papers/2605.22791, the Gated Delta Rule-2 paragraph), with
// KBE = K*B*E, QE = Q*E, KiE = K/E, E = exp(G), E_C = exp(G_C):
//     R = W_gate*V - KBE S^T,      U = T R
//     dU = KiE (D Diag(E_C))^T + P^T dO,   dR = T^T dU
//     dA = -dR U^T (strict lower), dP = dO U^T (lower)
//     dv = w * dR,  dw = v * dR
//     dKBE = -dR S + dA KiE,   dQE = dO S + dP KiE,
//     dKiE = (U D) Diag(E_C) + dA^T KBE + dP^T QE,
//     dE_C = colsum((U D) * KiE) + colsum(S * D),
// then the chain rule through the gates, token by token:
//     dk = dKBE B E + dKiE / E,  db = dKBE K E,  dq = dQE E,
//     dG = dKBE KBE + dQE QE - dKiE KiE,
// and dlog alpha_r = E_C dE_C + the sum of dG over tokens r .. C-1.
// KiE (D Diag(E_C))^T is the product D (K*exp(G_C - G))^T; with the scaled
// D' = D Diag(E_C), U D' is (U D) Diag(E_C) directly.  Every product has the
// channel on M = 128 (TMEM lane); four MMA groups:
//   G1  X = S KBE^T (-> R^T),  S^T dO^T,  dU^T = D' KiE^T + dO^T P
//   G2  U^T = R^T T^T,  dR^T = dU^T T
//   G3  [dA'; dP] = [dR; dO] U^T,  -S^T dR^T,  D'^T U^T
//   G4  [dKBE^T | dQE^T] += KiE^T [dA; dP]^T,  dKiE^T += KBE^T dA + QE^T dP
// A chunk decaying past e^20 (where the bf16 factors would span more than
// that) only gets its mode written; the CUDA-core reverse pass and the chunk
// kernel (bwd2_tc.cuh) take it.
#pragma once
#include <cuda.h>

#include "bwd2_tc.cuh"
#include "common.cuh"
#include "fwd2_tc2.cuh"
#include "sm100.cuh"

namespace gdr {

constexpr int kG2gThreads = 512;

struct G2gLayout {
    static constexpr uint32_t K = 0;          // K tile (TMA) [r][j], 2 halves x 8 KB; then dU^T [c][r]
    static constexpr uint32_t V = 16384;      // V tile (TMA) [r][c]; then fixed-order sums [4][128] fp32
    static constexpr uint32_t DOR = 32768;    // per c half (16 KB): dR rows at +0, dO rows (TMA) at +8192
    static constexpr uint32_t S = 65536;      // S bf16 [c][j], 2 halves x 16 KB; then [dA; dP] bf16 [r'][i]
    static constexpr uint32_t D = 98304;      // D Diag(E_C) bf16 [c][j]; then Q*E [r][j]
    static constexpr uint32_t KB = 131072;    // K*B*E [r][j]
    static constexpr uint32_t KI = 147456;    // scan partials; then K/E [r][j]
    static constexpr uint32_t RU = 163840;    // R^T, then U^T, [c][r]
    static constexpr uint32_t TB = 180224;    // T bf16 [r][i]
    static constexpr uint32_t PB = 188416;    // P bf16 [r][i]
    static constexpr uint32_t G = 196608;     // log alpha [64][128] fp32 (TMA), scanned in place into G
    static constexpr uint32_t EC = G + 32768;  // E_C [128], dE_C [128] fp32, the mode code
    static constexpr uint32_t BAR = EC + 1040;
    static constexpr uint32_t BYTES = BAR + 64;
    static constexpr uint32_t kAlloc = BYTES + 1024;
};
static_assert(G2gLayout::kAlloc <= 232448, "shared memory budget");
static_assert(G2gLayout::BAR % 8 == 0, "barrier alignment");

// TMEM columns (512 allocated): lanes = value channel c for X, dU, U, dR; row
// r' of [dA'; dP] for AP; key channel j for KB, QE (adjacent, for G4's N = 128
// product) and UD
constexpr uint32_t kG2gX = 0, kG2gAP = 64, kG2gDU = 128, kG2gU = 192, kG2gDR = 256, kG2gKB = 320,
                   kG2gQE = 384, kG2gUD = 448;

__global__ void __launch_bounds__(kG2gThreads, 1)
gdr2_bwd_grad_tc_kernel(const __grid_constant__ CUtensorMap tm_k, const __grid_constant__ CUtensorMap tm_v,
                        const __grid_constant__ CUtensorMap tm_do, const __grid_constant__ CUtensorMap tm_la,
                        int T, int H, const __nv_bfloat16 *__restrict__ qg, const __nv_bfloat16 *__restrict__ kg,
                        const float *__restrict__ bgate, const float *__restrict__ wgate,
                        const float *__restrict__ S_chunks, const float *__restrict__ D_chunks,
                        const float *__restrict__ TP, __nv_bfloat16 *__restrict__ dq_out,
                        __nv_bfloat16 *__restrict__ dk_out, __nv_bfloat16 *__restrict__ dv_out,
                        float *__restrict__ dla_out, float *__restrict__ db_out, float *__restrict__ dw_out,
                        int *__restrict__ exact_flags, int *__restrict__ todo, int *__restrict__ ntodo) {
    using L = G2gLayout;
    using namespace sm100;
    constexpr int DK = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4, 16 columns each)
    const int row = wq * 32 + lane;           // TMEM lane
    const int nch = (T + kChunk - 1) / kChunk;
    const int ch = blockIdx.x % nch, bh = blockIdx.x / nch, b = bh / H, h = bh % H;
    const int t0 = ch * kChunk, nv = min(kChunk, T - t0);
    const size_t tok0 = ((size_t)b * T + t0) * H + h;
    const size_t tile = (size_t)bh * nch + ch;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR), *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *sg = reinterpret_cast<float *>(sm + L::G), *ec = reinterpret_cast<float *>(sm + L::EC);
    float *dec_s = ec + 128;
    int *code = reinterpret_cast<int *>(ec + 256);
    float *scan = reinterpret_cast<float *>(sm + L::KI);
    float *red = reinterpret_cast<float *>(sm + L::V);
    const uint32_t sbase = smem_u32(sm);
    auto tok = [&](int r) { return tok0 + (size_t)r * H; };

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *abort_flag = 0;
        *code = 0;
        mbar_expect_tx(bar_tma, 3 * 16384 + 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(sm + L::K + half * 8192, &tm_k, bar_tma, half * 64, h, t0, b);
            tma_load_4d(sm + L::V + half * 8192, &tm_v, bar_tma, half * 64, h, t0, b);
            tma_load_4d(sm + L::DOR + half * 16384 + 8192, &tm_do, bar_tma, half * 64, h, t0, b);
        }
        tma_load_4d(sm + L::G, &tm_la, bar_tma, 0, h, t0, b);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    // D (read after the scan) and this chunk's q rows -> L2
    prefetch_l2(D_chunks + tile * DK * DK + 32 * tid);
    if (tid < 2 * kChunk && (tid >> 1) < nv) prefetch_l2(qg + tok(tid >> 1) * DK + 64 * (tid & 1));
    // this thread's w (rows 16 wc .. 16 wc + 15 of value channel `row`) and b (two tile items)
    float wv[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
        const int r = wc * 16 + i;
        wv[i] = r < nv ? wgate[tok(r) * DK + row] : 0.f;
    }
    float bq[2][8];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int item = tid + m * kG2gThreads, r = item >> 4, c8 = (item & 15) * 8;
        if (r < nv) load8(bgate + tok(r) * DK + c8, bq[m]);
        else
#pragma unroll
            for (int i = 0; i < 8; ++i) bq[m][i] = 0.f;
    }
    // S (fp32 [c][j]) -> bf16 K-major tile; T and P (fp32 [r][i]) -> bf16
#pragma unroll 2
    for (int m = 0; m < 4; ++m) {
        const int item = tid + m * kG2gThreads, c = item >> 4, j8 = (item & 15) * 8;
        float x[8];
        load8(S_chunks + (tile * DK + c) * DK + j8, x);
        st_bf16x8(sm + L::S + (j8 >> 6) * 16384 + sw128_offset(c, (j8 & 63) >> 3), x);
    }
    {
        const int r = tid >> 3, i8 = (tid & 7) * 8;
        const float *tp = TP + tile * 2 * kChunk * kChunk;
        float x[8];
        load8(tp + r * kChunk + i8, x);
        st_bf16x8(sm + L::TB + sw128_offset(r, i8 >> 3), x);
        load8(tp + kChunk * kChunk + r * kChunk + i8, x);
        st_bf16x8(sm + L::PB + sw128_offset(r, i8 >> 3), x);
    }
    bool tma_pending = true;  // thread 0
    if (tid == 0) {
        if (!mbar_wait(bar_tma, 0)) *abort_flag = 1;
        else tma_pending = false;
    }
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);

    // per-channel scan of log alpha in place (channel j = tid % 128, rows
    // 16 rg .. 16 rg + 15), E_C, and the chunk's mode
    if (!*abort_flag) {
        const int j = tid & 127, rg = tid >> 7;
        float g[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) g[i] = sg[(rg * 16 + i) * DK + j];  // rows past T read as zero
#pragma unroll
        for (int i = 1; i < 16; ++i) g[i] += g[i - 1];
        scan[rg * DK + j] = g[15];
        __syncthreads();
        float off = 0.f, tot = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x = scan[q * DK + j];
            off += q < rg ? x : 0.f;
            tot += x;
        }
        if (rg == 0) {
            ec[j] = expf(tot);
            if (-tot > 80.f) atomicMax(code, 2);
            else if (-tot > kBwd2TcSpan) atomicMax(code, 1);
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sg[(rg * 16 + i) * DK + j] = g[i] + off;
    }
    __syncthreads();
    const int mode = *code == 2 ? kChunkExact : *code == 1 ? kChunkF32 : kChunkTc;
    if (tid == 0) {
        exact_flags[tile] = mode;
        if (mode != kChunkTc) todo[atomicAdd(ntodo, 1)] = (int)tile;  // left to the CUDA-core pass
    }
    const bool work = mode == kChunkTc && !*abort_flag;

    if (work) {
        // K*B*E and K/E: two items of 8 channels per thread
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int item = tid + m * kG2gThreads, r = item >> 4, c8 = (item & 15) * 8;
            const uint32_t off = (c8 >> 6) * 8192 + sw128_offset(r, (c8 & 63) >> 3);
            float G[8], kk[8], kbe[8], kie[8];
            load8(sg + r * DK + c8, G);
            load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::K + off), kk);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float e = __expf(G[i]);
                kbe[i] = kk[i] * bq[m][i] * e;
                kie[i] = __fdividef(kk[i], e);
            }
            st_bf16x8(sm + L::KB + off, kbe);
            st_bf16x8(sm + L::KI + off, kie);
        }
        // D Diag(E_C) -> bf16 K-major tile
#pragma unroll 2
        for (int m = 0; m < 4; ++m) {
            const int item = tid + m * kG2gThreads, c = item >> 4, j8 = (item & 15) * 8;
            float x[8], e8[8];
            load8(D_chunks + (tile * DK + c) * DK + j8, x);
            load8(ec + j8, e8);
#pragma unroll
            for (int i = 0; i < 8; ++i) x[i] *= e8[i];
            st_bf16x8(sm + L::D + (j8 >> 6) * 16384 + sw128_offset(c, (j8 & 63) >> 3), x);
        }
    }
    fence_async_smem();
    tc_before_sync();
    __syncthreads();

    uint32_t mph = 0;
    auto mma_done = [&]() -> bool {  // every thread: the last commit of bar_mma has completed
        if (tid == 0 && !*abort_flag && !mbar_wait(bar_mma, mph)) *abort_flag = 1;
        mph ^= 1;
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
        return *abort_flag == 0;
    };
    const uint32_t sS = sbase + L::S, sD = sbase + L::D, sKB = sbase + L::KB, sKI = sbase + L::KI;
    const uint32_t sRU = sbase + L::RU, sT = sbase + L::TB, sP = sbase + L::PB, sDOR = sbase + L::DOR;
    const uint32_t sDU = sbase + L::K;
    int ncommit = 0;
    do {
        if (!work) break;
        // ---- G1
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // X = S KBE^T
                mma_bf16(tmem + kG2gX, smem_desc_sw128(sS + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(sKB + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // S^T dO^T
                mma_bf16(tmem + kG2gQE, smem_desc_sw128(sS + kk * 2048, 16384, 1024),
                         smem_desc_sw128(sDOR + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, true, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)  // dU^T = D' KiE^T ...
                mma_bf16(tmem + kG2gDU, smem_desc_sw128(sD + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(sKI + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // ... + dO^T P
                mma_bf16(tmem + kG2gDU, smem_desc_sw128(sDOR + 8192 + kk * 2048, 16384, 1024),
                         smem_desc_sw128(sP + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), 1);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_done()) break;
        {   // R^T = W_gate*V^T - X -> bf16 [c][r]; dU^T -> bf16 [c][r] over K's tile
            const int c = row;
            const uint8_t *vh = sm + L::V + (c >> 6) * 8192;
            float x[16], du[16];
            tmem_ld16x2(tl + kG2gX + wc * 16, x, tl + kG2gDU + wc * 16, du);
#pragma unroll
            for (int i = 0; i < 16; ++i) x[i] = wv[i] * ld_sw_bf16(vh, wc * 16 + i, c & 63) - x[i];
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) {
                st_bf16x8(sm + L::RU + sw128_offset(c, wc * 2 + q2), x + 8 * q2);
                st_bf16x8(sm + L::K + sw128_offset(c, wc * 2 + q2), du + 8 * q2);
            }
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // ---- G2: U^T = R^T T^T, dR^T = dU^T T
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2gU, smem_desc_sw128(sRU + kk * 32, 16, 1024), smem_desc_sw128(sT + kk * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2gDR, smem_desc_sw128(sDU + kk * 32, 16, 1024),
                         smem_desc_sw128(sT + kk * 2048, 8192, 1024), idesc_bf16(128, 64, false, true), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_done()) break;
        {   // U^T -> bf16 [c][r] over R^T; dR -> bf16 [r][c] in [dR; dO]; dv = w dR, dw = v dR
            const int c = row;
            float u[16], dr[16];
            tmem_ld16x2(tl + kG2gU + wc * 16, u, tl + kG2gDR + wc * 16, dr);
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) st_bf16x8(sm + L::RU + sw128_offset(c, wc * 2 + q2), u + 8 * q2);
            uint8_t *drh = sm + L::DOR + (c >> 6) * 16384;
            const uint8_t *vh = sm + L::V + (c >> 6) * 8192;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = wc * 16 + i;
                st_sw_bf16(drh, r, c & 63, dr[i]);
                if (r < nv) {
                    const size_t off = tok(r) * DK + c;
                    dv_out[off] = __float2bfloat16_rn(wv[i] * dr[i]);
                    dw_out[off] = ld_sw_bf16(vh, r, c & 63) * dr[i];
                }
            }
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // ---- G3: [dA'; dP] = [dR; dO] U^T, -S^T dR^T, D'^T U^T
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2gAP, smem_desc_sw128(sDOR + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(sRU + kk * 2048, 8192, 1024), idesc_bf16(128, 64, false, true), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2gKB, smem_desc_sw128(sS + kk * 2048, 16384, 1024),
                         smem_desc_sw128(sDOR + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, true, false, true), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2gUD, smem_desc_sw128(sD + kk * 2048, 16384, 1024),
                         smem_desc_sw128(sRU + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_done()) break;
        {   // [dA; dP] -> bf16 [r'][i] over S (dA = -dA' strictly lower, dP lower)
            float v[16];
            tmem_ld16(tl + kG2gAP + wc * 16, v);
            const int i0 = wc * 16;
            if (row < 64) {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = (i0 + i < row) ? -v[i] : 0.f;
            } else {
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = (i0 + i <= row - 64) ? v[i] : 0.f;
            }
#pragma unroll
            for (int q2 = 0; q2 < 2; ++q2) st_bf16x8(sm + L::S + sw128_offset(row, wc * 2 + q2), v + 8 * q2);
        }
        {   // dE_C, channel j = row: colsum((U D) KiE) over this thread's 16 tokens
            // (U D' = (U D) E_C) and colsum(S D) over its 32 value rows (fp32 S and D)
            const int j = row;
            float ud[16];
            tmem_ld16(tl + kG2gUD + wc * 16, ud);
            const uint8_t *kih = sm + L::KI + (j >> 6) * 8192;
            float a = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) a = fmaf(ud[i], ld_sw_bf16(kih, wc * 16 + i, j & 63), a);
            float sd = 0.f;
            const float *sp = S_chunks + tile * DK * DK, *dp = D_chunks + tile * DK * DK;
#pragma unroll 8
            for (int c = wc * 32; c < wc * 32 + 32; ++c) sd = fmaf(sp[c * DK + j], dp[c * DK + j], sd);
            red[wc * DK + j] = __fdividef(a, ec[j]) + sd;
        }
        // Q*E -> bf16 [r][j] over D' (two items of 8 channels per thread)
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int item = tid + m * kG2gThreads, r = item >> 4, c8 = (item & 15) * 8;
            const uint32_t off = (c8 >> 6) * 8192 + sw128_offset(r, (c8 & 63) >> 3);
            float G[8], qq[8];
            load8(sg + r * DK + c8, G);
            if (r < nv) load8(qg + tok(r) * DK + c8, qq);
            else
#pragma unroll
                for (int i = 0; i < 8; ++i) qq[i] = 0.f;
#pragma unroll
            for (int i = 0; i < 8; ++i) qq[i] *= __expf(G[i]);
            st_bf16x8(sm + L::D + off, qq);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();
        if (tid < DK) dec_s[tid] = red[tid] + red[DK + tid] + red[2 * DK + tid] + red[3 * DK + tid];

        // ---- G4: [dKBE^T | dQE^T] += KiE^T [dA; dP]^T, dKiE^T += KBE^T dA + QE^T dP
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2gKB, smem_desc_sw128(sKI + kk * 2048, 8192, 1024),
                         smem_desc_sw128(sS + kk * 32, 16, 1024), idesc_bf16(128, 128, true, false), 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2gUD, smem_desc_sw128(sKB + kk * 2048, 8192, 1024),
                         smem_desc_sw128(sS + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2gUD, smem_desc_sw128(sD + kk * 2048, 8192, 1024),
                         smem_desc_sw128(sS + 8192 + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true), 1);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_done()) break;
        {   // the chain rule through the gates, channel j = row, tokens 16 wc .. 16 wc + 15;
            // dlog alpha as the in-chunk suffix sum of dG (later groups first) plus E_C dE_C
            const int j = row;
            float skb[16], sqe[16], ski[16];
            tmem_ld16x2(tl + kG2gKB + wc * 16, skb, tl + kG2gQE + wc * 16, sqe);
            tmem_ld16(tl + kG2gUD + wc * 16, ski);
            float tot = 0.f;
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const int r = wc * 16 + i;
                float dg = 0.f;
                if (r < nv) {
                    const size_t off = tok(r) * DK + j;
                    const float e = __expf(sg[r * DK + j]), ie = __fdividef(1.f, e);
                    const float kv = __bfloat162float(kg[off]), qv = __bfloat162float(qg[off]), bv = bgate[off];
                    dk_out[off] = __float2bfloat16_rn(fmaf(skb[i] * bv, e, ski[i] * ie));
                    db_out[off] = skb[i] * kv * e;
                    dq_out[off] = __float2bfloat16_rn(sqe[i] * e);
                    dg = skb[i] * kv * bv * e + sqe[i] * qv * e - ski[i] * kv * ie;
                }
                skb[i] = dg;
                tot += dg;
            }
            __syncthreads();  // `red` (dE_C's sums) is consumed
            red[wc * DK + j] = tot;
            __syncthreads();
            float suffix = ec[j] * dec_s[j];  // dG_C, carried to every token of the chunk
#pragma unroll
            for (int u = 3; u > 0; --u)
                if (u > wc) suffix += red[u * DK + j];
#pragma unroll
            for (int i = 15; i >= 0; --i) {
                const int r = wc * 16 + i;
                suffix += skb[i];
                if (r < nv) dla_out[tok(r) * DK + j] = suffix;
            }
        }
    } while (0);

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

// One CTA per (b, h, chunk): all gradients of the chunks it takes (mode 0);
// the others get their mode in `flags` and are appended to todo (*ntodo,
// zeroed by the caller, counts them) for the CUDA-core reverse pass and the
// chunk kernel.
inline cudaError_t launch_bwd2_grad_tc(int B, int T, int H, const void *q, const void *k, const void *v,
                                       const void *dO, const float *la, const float *bgate, const float *wgate,
                                       const float *S_chunks, const float *D_chunks, const float *TP, void *dq,
                                       void *dk, void *dv, float *dla, float *db, float *dw, int *flags,
                                       int *todo, int *ntodo, cudaStream_t stream) {
    CUtensorMap mk, mv, mdo, mla;
    if (!make_token_map(&mk, k, B, T, H, 128) || !make_token_map(&mv, v, B, T, H, 128) ||
        !make_token_map(&mdo, dO, B, T, H, 128) || !make_gate_map(&mla, la, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr2_bwd_grad_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)G2gLayout::kAlloc);
    if (err != cudaSuccess) return err;
    const int nch = (T + kChunk - 1) / kChunk;
    gdr2_bwd_grad_tc_kernel<<<(unsigned)(B * H * nch), kG2gThreads, G2gLayout::kAlloc, stream>>>(
        mk, mv, mdo, mla, T, H, static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(k),
        bgate, wgate, S_chunks, D_chunks, TP, static_cast<__nv_bfloat16 *>(dq), static_cast<__nv_bfloat16 *>(dk),
        static_cast<__nv_bfloat16 *>(dv), dla, db, dw, flags, todo, ntodo);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
