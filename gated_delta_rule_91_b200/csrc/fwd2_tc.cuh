// fwd2_tc.cuh -- chunkwise Gated DeltaNet-2 forward on the tensor cores
// (bf16 q/k/v/o, dk = dv = 128; fp32 gates, state and accumulation).
//
// Gated Delta Rule-2 ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
// Attention", agihunt.info/papers/2605.22791, the Gated Delta Rule-2
// paragraph): per token, decay each key channel by alpha_t, read along
// b_t*k_t, write the residual of w_t*v_t along k_t.  Chunkwise (the form
// restated in gdr2_simt.cuh), with per-channel cumulative log decay
// G_r[j] = sum_{s<=r} log alpha_s[j] inside a 64-token chunk and E = exp(G):
//     A = strictLower((K*B*E)(K/E)^T),  P = inclLower((Q*E)(K/E)^T),  T = (I + A)^{-1}
//     W = T (K*B*E),  U = T (W_gate*V) - W S^T
//     O = (Q*E) S^T + P U,   S <- S Diag(E_C) + U^T (K * exp(G_C - G)).
// Every operand except K/E is bounded by the inputs (E <= 1, exp(G_C - G) <= 1).
// K/E only feeds A and P; a chunk in which some channel decays by more than
// e^80 (where K/E could overflow) evaluates A and P exactly on CUDA cores,
// term by term with exp(G_r[j] - G_i[j]).
//
// One CTA of 512 threads per (b, h), the fp32 state in TMEM.  Per chunk:
//  1. gates and operand tiles on CUDA cores: the per-channel scan of
//     log alpha (4 row groups x 128 channels), then bf16 tiles K*B*E and Q*E
//     (stacked as the M = 128 A operand of step 2), K/E, K*exp(G_C - G) and
//     W_gate*V, 128B-swizzled like the TMA tiles they come from;
//  2. one tcgen05 MMA [K*B*E; Q*E](K/E)^T gives A and P;
//  3. the inverse T on two warps (as in the scalar-gate kernel) while the
//     other warps turn S into its bf16 operand and scale S by exp(G_C);
//  4. W^T = (K*B*E)^T T^T and U^gT = (W_gate*V)^T T^T, then U^T -= S W^T and
//     O^T = S (Q*E)^T;
//  5. O^T += U^T P^T, S += U^T (K*exp(G_C - G)); O leaves through a TMA store.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "fwd_tc.cuh"
#include "fwd_tc2.cuh"
#include "sm100.cuh"

namespace gdr {

constexpr int kG2Threads = 512;

struct G2Layout {
    static constexpr uint32_t TK = 0;         // TMA K tile, 2 halves x 8 KB
    static constexpr uint32_t TQ = 16384;     // TMA Q tile
    static constexpr uint32_t TV = 32768;     // TMA V tile
    static constexpr uint32_t KQE = 49152;    // [K*B*E; Q*E] per dk half: K*B*E rows at +0, Q*E at +8192
    static constexpr uint32_t KIE = 81920;    // K/E [r][j]; then W [j][r] (MN-major B of U^T -= S W^T)
    static constexpr uint32_t KTL = 98304;    // K * exp(G_C - G) [r][j]
    static constexpr uint32_t WV = 114688;    // W_gate * V [r][c]; then U^T [c][r]
    static constexpr uint32_t SB = 131072;    // S bf16 [c][j] (2 halves x 16 KB); G fp32 scratch of the exact path
    static constexpr uint32_t TB = 163840;    // T bf16 [r][i]
    static constexpr uint32_t PB = 172032;    // P bf16 [r][i]
    static constexpr uint32_t FA = 180224;    // A fp32 (64 x kLdT)
    static constexpr uint32_t FT = FA + 64 * kLdT * 4;    // T fp32; later the O tile of the TMA store
    static constexpr uint32_t OST = (FT + 1023) / 1024 * 1024;
    static constexpr uint32_t MISC = FT + 64 * kLdT * 4;  // E_C[128], scan partials [4][128], ones[64], flag
    static constexpr uint32_t BAR = MISC + (128 + 512 + 64 + 4) * 4;
    static constexpr uint32_t BYTES = BAR + 64;
    static constexpr uint32_t kAlloc = BYTES + 1024;
};
static_assert(G2Layout::OST + 16384 <= G2Layout::MISC, "O tile fits in the T scratch");
static_assert(G2Layout::kAlloc <= 232448, "shared memory budget");

// TMEM columns (512 allocated)
constexpr uint32_t kG2S = 0, kG2AP = 128, kG2W = 192, kG2U = 256, kG2O = 320;

// Step 1 for the chunk at tok0 (nv valid tokens), in two passes.
// Scan: thread (j = tid % 128, row group rg = tid / 128) takes channel j of
// rows 16 rg .. 16 rg + 15 and writes G (fp32 [r][j], into the S operand's
// space, which is free until step 3; the exact path reads it too), E_C and
// the chunk's exact-path flag (cleared by the caller).
// Tiles: thread items (row r, 8 channels) build 16 bytes of every operand
// tile at once, at the swizzled position of the TMA tile they come from.
__device__ __forceinline__ void g2_tiles(uint8_t *sm, const float *log_alpha, const float *bgate,
                                         const float *wgate, size_t tok0, int H, int nv) {
    using L = G2Layout;
    using namespace sm100;
    const int tid = threadIdx.x;
    float *ec = reinterpret_cast<float *>(sm + L::MISC), *scan = ec + 128;
    volatile int *flag = reinterpret_cast<volatile int *>(ec + 128 + 512 + 64);
    float *sg = reinterpret_cast<float *>(sm + L::SB);
    // the b and w gates of this thread's two tile items are loaded first, so
    // their latency overlaps the scan's
    float4 bq[2][2], wq[2][2];
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int item = tid + m * kG2Threads, r = item >> 4, c8 = (item & 15) * 8;
        const size_t e = (tok0 + (size_t)r * H) * 128 + c8;
        const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
        bq[m][0] = r < nv ? *reinterpret_cast<const float4 *>(bgate + e) : z;
        bq[m][1] = r < nv ? *reinterpret_cast<const float4 *>(bgate + e + 4) : z;
        wq[m][0] = r < nv ? *reinterpret_cast<const float4 *>(wgate + e) : z;
        wq[m][1] = r < nv ? *reinterpret_cast<const float4 *>(wgate + e + 4) : z;
    }
    {
        const int j = tid & 127, rg = tid >> 7;
        float g[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
            const int r = rg * 16 + i;
            g[i] = r < nv ? log_alpha[(tok0 + (size_t)r * H) * 128 + j] : 0.f;
        }
#pragma unroll
        for (int i = 1; i < 16; ++i) g[i] += g[i - 1];
        scan[rg * 128 + j] = g[15];
        __syncthreads();
        float off = 0.f, tot = 0.f;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
            const float x = scan[q * 128 + j];
            off += q < rg ? x : 0.f;
            tot += x;
        }
        if (rg == 0) {
            ec[j] = expf(tot);
            if (-tot > 80.f) *flag = 1;
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) sg[(rg * 16 + i) * 128 + j] = g[i] + off;
    }
    __syncthreads();
#pragma unroll
    for (int m = 0; m < 2; ++m) {
        const int item = tid + m * kG2Threads, r = item >> 4, c8 = (item & 15) * 8;
        const int hj = c8 >> 6;
        const uint32_t off = sw128_offset(r, (c8 & 63) >> 3);
        float G[8], Gc[8], kk[8], qq[8], vv[8];
        const bool exact = *flag != 0;
        const float bb[8] = {bq[m][0].x, bq[m][0].y, bq[m][0].z, bq[m][0].w,
                             bq[m][1].x, bq[m][1].y, bq[m][1].z, bq[m][1].w};
        const float ww[8] = {wq[m][0].x, wq[m][0].y, wq[m][0].z, wq[m][0].w,
                             wq[m][1].x, wq[m][1].y, wq[m][1].z, wq[m][1].w};
        load8(sg + r * 128 + c8, G);
        load8(sg + 63 * 128 + c8, Gc);
        load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::TK + hj * 8192 + off), kk);
        load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::TQ + hj * 8192 + off), qq);
        load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::TV + hj * 8192 + off), vv);
        float kbe[8], qe[8], kie[8], ktl[8], wv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const float e = __expf(G[i]);
            kbe[i] = kk[i] * bb[i] * e;
            qe[i] = qq[i] * e;
            kie[i] = -G[i] <= 80.f ? __fdividef(kk[i], e) : 0.f;
            wv[i] = ww[i] * vv[i];
        }
        if (!exact) {  // K exp(G_C - G) = (K/E) exp(G_C), with E_C = exp(G_C) <= 1
            const float4 e0 = *reinterpret_cast<const float4 *>(ec + c8), e1 = *reinterpret_cast<const float4 *>(ec + c8 + 4);
            const float ecv[8] = {e0.x, e0.y, e0.z, e0.w, e1.x, e1.y, e1.z, e1.w};
#pragma unroll
            for (int i = 0; i < 8; ++i) ktl[i] = kie[i] * ecv[i];
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) ktl[i] = kk[i] * __expf(Gc[i] - G[i]);
        }
        st_bf16x8(sm + L::KQE + hj * 16384 + off, kbe);
        st_bf16x8(sm + L::KQE + hj * 16384 + 8192 + off, qe);
        st_bf16x8(sm + L::KIE + hj * 8192 + off, kie);
        st_bf16x8(sm + L::KTL + hj * 8192 + off, ktl);
        st_bf16x8(sm + L::WV + hj * 8192 + off, wv);
    }
}

__global__ void __launch_bounds__(kG2Threads, 1)
gdr2_fwd_tc_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                   int T, int H, const float *__restrict__ log_alpha, const float *__restrict__ bgate,
                   const float *__restrict__ wgate, const float *__restrict__ S0, float *__restrict__ S_T,
                   int store_o, float *__restrict__ S_chunks, float *__restrict__ TP_chunks) {
    using L = G2Layout;
    using namespace sm100;
    constexpr int D = 128;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;           // TMEM lane
    const int bh = blockIdx.x, b = bh / H, h = bh % H;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR), *bar_mma = bar_tma + 1;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 2);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *ec = reinterpret_cast<float *>(sm + L::MISC), *ones = ec + 128 + 512;
    volatile int *xflag = reinterpret_cast<volatile int *>(ones + 64);
    float *sA = reinterpret_cast<float *>(sm + L::FA), *sT = reinterpret_cast<float *>(sm + L::FT);
    const uint32_t sbase = smem_u32(sm);
    const uint32_t kqe = sbase + L::KQE, kie = sbase + L::KIE, ktl = sbase + L::KTL, wv = sbase + L::WV;
    const uint32_t sb = sbase + L::SB, tb = sbase + L::TB, pb = sbase + L::PB;

    if (tid == 0) {
        mbar_init(bar_tma, 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(&tm_q);
        prefetch_tmap(&tm_k);
        prefetch_tmap(&tm_v);
        prefetch_tmap(&tm_o);
    }
    if (tid < 64) ones[tid] = 1.f;
    // T's bf16 tile: the inverse writes only its lower triangle, so zero it once
    for (int k = tid; k < 512; k += kG2Threads)
        *reinterpret_cast<uint4 *>(sm + L::TB + k * 16) = make_uint4(0, 0, 0, 0);
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    {   // entry state -> TMEM (row `row`, this column group's 32 columns)
        float v[32];
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
        tmem_st32(tl + kG2S + col, v);
        tmem_wait_st();
    }

    uint32_t tph = 0, mph = 0;
    int ncommit = 0;  // commits of bar_mma (thread 0)
    bool tma_pending = false;
    auto issue_tma = [&](int n) {
        mbar_expect_tx(bar_tma, 49152);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(sm + L::TK + half * 8192, &tm_k, bar_tma, half * 64, h, n * kChunk, b);
            tma_load_4d(sm + L::TQ + half * 8192, &tm_q, bar_tma, half * 64, h, n * kChunk, b);
            tma_load_4d(sm + L::TV + half * 8192, &tm_v, bar_tma, half * 64, h, n * kChunk, b);
        }
    };
    auto mma_wait_all = [&]() -> bool {  // every thread: the last commit of bar_mma has completed
        if (tid == 0 && !*abort_flag && !mbar_wait(bar_mma, mph)) *abort_flag = 1;
        mph ^= 1;
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
        return *abort_flag == 0;
    };
    auto operands_ready = [&]() {  // shared-memory operands written by threads -> tensor cores
        fence_async_smem();
        tc_before_sync();
        __syncthreads();
    };
    if (tid == 0) {
        issue_tma(0);
        tma_pending = true;
    }

#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        const int t0 = n * kChunk, nv = min(kChunk, T - t0);
        const size_t tok0 = ((size_t)b * T + t0) * H + h;
        if (tid == 0) {
            *xflag = 0;
            if (!mbar_wait(bar_tma, tph)) *abort_flag = 1;
            else tma_pending = false;
        }
        tph ^= 1;
        __syncthreads();
        if (*abort_flag) break;

        // 1. gates and operand tiles
        g2_tiles(sm, log_alpha, bgate, wgate, tok0, H, nv);
        if (n + 1 < nch) {  // the next chunk's gate rows -> L2 (3 gates x 64 rows x 4 lines of 128 B)
            const int nv1 = min(kChunk, T - t0 - kChunk);
            for (int k = tid; k < 3 * 64 * 4; k += kG2Threads) {
                const int gate = k >> 8, r = (k >> 2) & 63, line = k & 3;
                if (r < nv1) {
                    const float *base = gate == 0 ? log_alpha : gate == 1 ? bgate : wgate;
                    prefetch_l2(base + (tok0 + (size_t)(kChunk + r) * H) * 128 + line * 32);
                }
            }
        }
        operands_ready();

        // 2. [K*B*E; Q*E] (K/E)^T -> A (rows 0-63), P (rows 64-127)
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2AP, smem_desc_sw128(kqe + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(kie + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;
        {
            float v[16];
            tmem_ld16(tl + kG2AP + wc * 16, v);
            const int i0 = wc * 16;
            if (row < 64) {
                const int r = row;
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = (i0 + i < r) ? v[i] : 0.f;
#pragma unroll
                for (int k4 = 0; k4 < 4; ++k4)
                    *reinterpret_cast<float4 *>(sA + r * kLdT + i0 + 4 * k4) =
                        make_float4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
            } else {
                const int r = row - 64;
#pragma unroll
                for (int i = 0; i < 16; ++i) v[i] = (i0 + i <= r) ? v[i] : 0.f;
#pragma unroll
                for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::PB + sw128_offset(r, wc * 2 + ch), v + 8 * ch);
                if (TP_chunks) {  // P in fp32 for the backward (second 64 x 64 block of the chunk)
                    float4 *dst = reinterpret_cast<float4 *>(
                        TP_chunks + (((size_t)bh * nch + n) * 2 + 1) * kChunk * kChunk + r * kChunk + i0);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        dst[k4] = make_float4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
                }
            }
        }
        __syncthreads();
        if (*xflag) {  // some channel decays past e^80 in this chunk: A and P term by term
            const float *sg = reinterpret_cast<const float *>(sm + L::SB);
            for (int p = tid; p < kChunk * kChunk; p += kG2Threads) {
                const int r = p >> 6, i = p & 63;
                if (i > r) continue;
                float a = 0.f, pq = 0.f;
                for (int jj = 0; jj < D; ++jj) {
                    const int hj = jj >> 6, cj = jj & 63;
                    const float kij = ld_sw_bf16(sm + L::TK + hj * 8192, i, cj) *
                                      __expf(sg[r * D + jj] - sg[i * D + jj]);
                    pq = fmaf(ld_sw_bf16(sm + L::TQ + hj * 8192, r, cj), kij, pq);
                    if (i < r && r < nv)
                        a = fmaf(ld_sw_bf16(sm + L::TK + hj * 8192, r, cj) * bgate[(tok0 + (size_t)r * H) * D + jj],
                                 kij, a);
                }
                if (i < r) sA[r * kLdT + i] = a;
                st_sw_bf16(sm + L::PB, r, i, pq);
            }
            __syncthreads();
        }
        // the raw tiles are consumed: next chunk's loads; the previous O tile has
        // to leave the T scratch it shares
        if (tid == 0) {
            if (n + 1 < nch) {
                issue_tma(n + 1);
                tma_pending = true;
            }
            bulk_wait_read_all();
        }
        __syncthreads();

        // 3. inverse (warps 0 and 1, also writing T in bf16); S -> bf16, S *= exp(G_C)
        if (warp < 2) inverse_two_warps(sA, sT, warp, lane, 1, TEmit{sm + L::TB, nullptr, ones, ones});
        {
            const int col = wc * 32;
            float v[32];
            tmem_ld32(tl + kG2S + col, v);
            if (S_chunks) {  // entry state of chunk n, fp32, for the backward's recompute
                float4 *dst = reinterpret_cast<float4 *>(S_chunks + (((size_t)bh * nch + n) * D + row) * D + col);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            uint8_t *half = sm + L::SB + (wc >> 1) * 16384;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) st_bf16x8(half + sw128_offset(row, (wc & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= ec[col + i];
            tmem_st32(tl + kG2S + col, v);
            tmem_wait_st();
        }
        operands_ready();

        // 4a. W^T = (K*B*E)^T T^T, U^gT = (W_gate*V)^T T^T
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2W, smem_desc_sw128(kqe + kk * 2048, 16384, 1024),
                         smem_desc_sw128(tb + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2U, smem_desc_sw128(wv + kk * 2048, 8192, 1024),
                         smem_desc_sw128(tb + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (TP_chunks) {  // T in fp32 for the backward (its upper triangle as zeros)
            float *dst = TP_chunks + ((size_t)bh * nch + n) * 2 * kChunk * kChunk;
            for (int idx = tid; idx < kChunk * kChunk; idx += kG2Threads) {
                const int r = idx >> 6, i = idx & 63;
                dst[idx] = i <= r ? sT[r * kLdT + i] : 0.f;
            }
        }
        if (!mma_wait_all()) break;
        {   // W^T (lane j, column r) -> W [j][r] bf16 over K/E
            float v[16];
            tmem_ld16(tl + kG2W + wc * 16, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::KIE + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
        }
        operands_ready();

        // 4b. U^T -= S W^T ; O^T = S (Q*E)^T
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2U, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(kie + kk * 2048, 8192, 1024), idesc_bf16(128, 64, false, true, true), 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2O, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(kqe + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;
        {   // U^T -> bf16 [c][r] over W_gate*V
            float v[16];
            tmem_ld16(tl + kG2U + wc * 16, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::WV + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
        }
        operands_ready();

        // 5. O^T += U^T P^T ; S += U^T (K * exp(G_C - G))
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2O, smem_desc_sw128(wv + kk * 32, 16, 1024), smem_desc_sw128(pb + kk * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2S, smem_desc_sw128(wv + kk * 32, 16, 1024),
                         smem_desc_sw128(ktl + kk * 2048, 8192, 1024), idesc_bf16(128, 128, false, true), 1);
            mma_commit(bar_mma);
            ++ncommit;
        }
        if (!mma_wait_all()) break;
        if (store_o) {  // O^T (lane = value channel, column = token) -> bf16 tile [token][channel]
            float v[16];
            tmem_ld16(tl + kG2O + wc * 16, v);
            uint8_t *half = sm + L::OST + (row >> 6) * 8192;
            const int cc = row & 63;
#pragma unroll
            for (int i = 0; i < 16; ++i) st_sw_bf16(half, wc * 16 + i, cc, v[i]);
        }
        fence_async_smem();
        __syncthreads();
        if (tid == 0 && store_o) {
            tma_store_4d(&tm_o, sm + L::OST, 0, h, t0, b);
            tma_store_4d(&tm_o, sm + L::OST + 8192, 64, h, t0, b);
            bulk_commit();
        }
    }

    if (!*abort_flag && S_T) {
        float v[32];
        const int col = wc * 32;
        tmem_ld32(tl + kG2S + col, v);
        float4 *dst = reinterpret_cast<float4 *>(S_T + ((size_t)bh * D + row) * D + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    if (tid == 0) bulk_wait_all();  // output stores complete before the CTA exits
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        if (tma_pending) mbar_wait(bar_tma, tph);
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

// TP_chunks (nullable) receives every chunk's T = (I + A)^{-1} and P in fp32,
// [B, H, nchunks, 2, 64, 64], for the backward's reverse pass.
// o == nullptr runs without outputs (the backward's recompute); S_chunks
// (nullable) receives every chunk's entry state, [B, H, nchunks, 128, 128] fp32.
inline cudaError_t launch_fwd2_tc(int B, int T, int H, const void *q, const void *k, const void *v,
                                  const float *la, const float *bgate, const float *wgate, const float *S0,
                                  void *o, float *S_T, cudaStream_t stream, float *S_chunks = nullptr,
                                  float *TP_chunks = nullptr) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128) || !make_token_map(&mo, o ? o : q, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr2_fwd_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)G2Layout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr2_fwd_tc_kernel<<<(unsigned)(B * H), kG2Threads, G2Layout::kAlloc, stream>>>(
        mq, mk, mv, mo, T, H, la, bgate, wgate, S0, S_T, o != nullptr ? 1 : 0, S_chunks, TP_chunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
