// fwd2_tc2.cuh -- the Gated DeltaNet-2 forward on a 2-CTA cluster per (b, h):
// a "prep" CTA and a "state" CTA on two SMs, 512 threads each.
//
// Same chunk algebra and operand orientation as fwd2_tc.cuh (Gated Delta
// Rule-2, "Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention",
// agihunt.info/papers/2605.22791; per-channel cumulative log decay G and
// E = exp(G) inside a 64-token chunk).  Everything that does not depend on the
// state S runs one chunk ahead on its own SM:
//
//   prep CTA (rank 0), per chunk n:
//     bf16 tiles K*B*E, Q*E (stacked as the M = 128 operand), K/E, K*exp(G_C - G)
//       from G (log alpha scanned per channel), b and the raw K/Q tiles
//     [K*B*E; Q*E] (K/E)^T (tcgen05)  ->  A = strictLower(.) (fp32), P = inclLower(.) (bf16)
//     T = (I + A)^{-1} on two warps (as in the scalar-gate kernels), while
//       eight other warps scan log alpha of chunk n+1 (-> G, E_C, exact-path flag)
//     -> two DSMEM bulk copies (64 KB of tiles, E_C) into the state's slot n % 2
//   state CTA (rank 1), per chunk n (fp32 S resident in TMEM):
//     W_gate*V from its own V tile, W^T = (K*B*E)^T T^T, U^gT = (W_gate*V)^T T^T
//                                             (built and issued one chunk ahead)
//     U^T -= S W^T,  O^T = S (Q*E)^T          (S read as bf16 operand)
//     O^T += U^T P^T,  S = S Diag(E_C) + U^T (K*exp(G_C - G))
//     O staged in shared memory and written by a TMA store.
// W of a chunk is written over that slot's K*B*E once W^T is formed; U^T is
// written over that chunk's W_gate*V.  A chunk in which some channel decays
// by more than e^80 forms A and P term by term on CUDA cores, as the
// single-CTA kernel does.
//
// Hand-off protocol (all waits bounded): the state CTA arms slot s with the
// byte count before the prep may copy into it, tells the prep with a remote
// mbarrier arrive ("landed") as soon as a copy has arrived, and gives the
// slot back with another ("empty") once every MMA of that chunk has
// completed.  The prep stages chunk n into its own slot n % 2 once the copy
// of chunk n - 2 out of it has landed, and copies chunk n out once the
// state's slot n % 2 is empty, so it can run up to two chunks ahead.  Both
// signals only report reads that are already complete (no data flows from
// the state CTA to the prep), so the prep polls them at CTA scope: a poll
// that acquires at cluster scope costs several hundred cycles even when the
// phase has completed.  No TMA multicast.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "fwd2_tc.cuh"
#include "fwd_tc2.cuh"
#include "sm100.cuh"

namespace gdr {

struct G2cLayout {
    // hand-off slot: identical offsets in the prep's staging slots and the state's slots.  The
    // prep loads the raw K and Q tiles straight into the slot and converts them in place; b
    // lands in the four 8 KB pieces the tiles overwrite last (K*B*E's halves, T and P).
    static constexpr uint32_t H_KQE = 0;      // [K*B*E; Q*E] per dk half: K*B*E at +0, Q*E (raw Q before) at +8192
    static constexpr uint32_t H_KTL = 32768;  // K * exp(G_C - G) [r][j] (raw K before)
    static constexpr uint32_t H_TB = 49152;   // T bf16 [r][i]  } K/E [r][j] (2 halves x 8 KB) until the
    static constexpr uint32_t H_PB = 57344;   // P bf16 [r][i]  } A/P product has read it
    static constexpr uint32_t H_TILES = 65536;
    static constexpr uint32_t H_EC = 512;     // E_C[128] fp32, copied from a region of its own
    static constexpr uint32_t H_BYTES = H_TILES + H_EC;
    // state CTA
    static constexpr uint32_t S_H = 0;                    // 2 slots of tiles
    static constexpr uint32_t S_EC = S_H + 2 * H_TILES;   // 2 x E_C
    static constexpr uint32_t S_V = S_EC + 2 * H_EC;      // V tile (TMA), 2 halves x 8 KB
    static constexpr uint32_t S_WV = S_V + 16384;         // 2 x (W_gate*V [r][c], then U^T [c][r])
    static constexpr uint32_t S_SB = S_WV + 2 * 16384;    // S bf16 [c][j], 2 halves x 16 KB
    static constexpr uint32_t S_OST = S_SB + 32768;       // O tile for the TMA store
    static constexpr uint32_t S_BAR = S_OST + 16384;
    static constexpr uint32_t S_BYTES = S_BAR + 128;
    // prep CTA
    static constexpr uint32_t P_STG = 0;                  // 2 staging slots of tiles
    static constexpr uint32_t P_EC = P_STG + 2 * H_TILES;  // 4 x E_C, by chunk mod 4
    static constexpr uint32_t P_LA = P_EC + 4 * H_EC;     // log alpha [64][128] fp32 (TMA), scanned in place into G
    static constexpr uint32_t P_AT = P_LA + 32768;        // A and T fp32 (64 x kLdT each)
    static constexpr uint32_t P_A = P_AT, P_T = P_AT + 64 * kLdT * 4;
    static constexpr uint32_t P_MISC = P_AT + 2 * 64 * kLdT * 4;  // scan partials [2][128], ones[64], flags, counts
    static constexpr uint32_t P_BAR = P_MISC + (256 + 64 + 16) * 4;
    static constexpr uint32_t P_BYTES = P_BAR + 128;
    static constexpr uint32_t kAlloc = (S_BYTES > P_BYTES ? S_BYTES : P_BYTES) + 1024;
};
static_assert(G2cLayout::S_V % 1024 == 0 && G2cLayout::S_WV % 1024 == 0 && G2cLayout::S_SB % 1024 == 0 &&
                  G2cLayout::S_OST % 1024 == 0 && G2cLayout::P_LA % 128 == 0,
              "TMA destinations: swizzled tiles 1024-aligned, plain tiles 128-aligned");
static_assert(G2cLayout::S_BAR % 8 == 0 && G2cLayout::P_BAR % 8 == 0, "barrier alignment");
static_assert(G2cLayout::kAlloc <= 232448, "shared memory budget");

// state TMEM columns (512 allocated): S, W^T, U^T x 2, O^T x 2
constexpr uint32_t kG2cS = 0, kG2cW = 128, kG2cU = 192, kG2cO = 320;
// prep barriers, in 8-byte words from P_BAR (the state CTA arrives on empty and landed)
constexpr uint32_t kG2cBarKq = 0, kG2cBarLa = 2, kG2cBarEmpty = 4, kG2cBarLanded = 6, kG2cBarMma = 8,
                   kG2cPrepBars = 9;
// prep roles: warps 0-1 solve the inverse; warps 8-15 scan the next chunk's
// log alpha meanwhile (named barrier 3); thread 32 issues the next chunk's
// loads while thread 0 waits for the A/P product
constexpr int kG2cScan0 = 256, kG2cScanThreads = 256, kG2cLoader = 32;

// ------------------------------------------------------------------ prep CTA --
// Per step n in staging slot s = n % 2: the raw K/Q tiles and b land in the
// slot (one TMA barrier per slot, issued one step ahead once the copy of
// step n-2 out of the slot has landed); log alpha lands in its own buffer
// during the previous step and is scanned there while that step's inverse
// runs.  k, q and b are also read from global memory by the exact path.
// Step n works on chunk n, or with `reverse` on chunk nch-1-n (the
// backward's dS pass); slots, buffers and parities follow the step.
__device__ __forceinline__ void g2c_prep(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                         const CUtensorMap *tm_la, const CUtensorMap *tm_bg, int T, int H, int b,
                                         int h, const __nv_bfloat16 *kg, const __nv_bfloat16 *qg,
                                         const float *bgate, float *TP_chunks, bool reverse = false) {
    using L = G2cLayout;
    using namespace sm100;
    constexpr int D = 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;           // TMEM lane
    const int bh = b * H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::P_BAR);
    uint64_t *tma_kq = bars + kG2cBarKq;  // [2]: raw K/Q and b of slot s
    uint64_t *tma_la = bars + kG2cBarLa;
    uint64_t *empty = bars + kG2cBarEmpty, *landed = bars + kG2cBarLanded;  // [2] each
    uint64_t *mma_bar = bars + kG2cBarMma;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kG2cPrepBars);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *scan = reinterpret_cast<float *>(sm + L::P_MISC), *ones = scan + 256;
    volatile int *xflag = reinterpret_cast<volatile int *>(ones + 64);  // [2], by chunk parity
    // TMA loads issued and waited for (for the drain after an abort): kq per slot, then la
    volatile int *kq_issued = xflag + 2, *kq_done = xflag + 4, *la_issued = xflag + 6, *la_done = xflag + 7;
    float *sg = reinterpret_cast<float *>(sm + L::P_LA);
    float *sA = reinterpret_cast<float *>(sm + L::P_A), *sT = reinterpret_cast<float *>(sm + L::P_T);
    auto ec_of = [&](int c) { return reinterpret_cast<float *>(sm + L::P_EC + (c & 3) * L::H_EC); };
    auto chunk_of = [&](int n) { return reverse ? nch - 1 - n : n; };
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        for (int i = 0; i < (int)kG2cPrepBars; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        *abort_flag = 0;
        for (int i = 0; i < 8; ++i) xflag[i] = 0;
        prefetch_tmap(tm_q);
        prefetch_tmap(tm_k);
        prefetch_tmap(tm_la);
        prefetch_tmap(tm_bg);
    }
    if (tid < 64) ones[tid] = 1.f;
    if (warp == 0) tmem_alloc(tmem_slot, 64);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    cluster_sync();  // both CTAs' barriers are initialised (and the state's slots armed)
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t remote_slot0 = cluster_addr(sm + L::S_H, 1);
    const uint32_t remote_ec0 = cluster_addr(sm + L::S_EC, 1);
    const uint32_t remote_full0 = cluster_addr(sm + L::S_BAR + 8, 1);  // state's hand_full[0]

    // raw K into the slot's K*exp(G_C - G) tile, raw Q into its Q*E rows, b
    // rows 16p .. 16p + 15 into piece p (K*B*E's two halves, T, P)
    auto issue_kq = [&](int n) {  // step n: slot n % 2, chunk chunk_of(n)
        const int sl = n & 1, t0 = chunk_of(n) * kChunk;
        uint8_t *st = sm + L::P_STG + sl * L::H_TILES;
        uint64_t *bar = &tma_kq[sl];
        mbar_expect_tx(bar, 65536);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(st + L::H_KTL + half * 8192, tm_k, bar, half * 64, h, t0, b);
            tma_load_4d(st + L::H_KQE + half * 16384 + 8192, tm_q, bar, half * 64, h, t0, b);
        }
        const uint32_t piece[4] = {L::H_KQE, L::H_KQE + 16384, L::H_TB, L::H_PB};
#pragma unroll
        for (int p = 0; p < 4; ++p) tma_load_4d(st + piece[p], tm_bg, bar, 0, h, t0 + 16 * p, b);
        kq_issued[sl] = kq_issued[sl] + 1;
    };
    auto issue_la = [&](int n) {
        mbar_expect_tx(tma_la, 32768);
        tma_load_4d(sm + L::P_LA, tm_la, tma_la, 0, h, chunk_of(n) * kChunk, b);
        *la_issued = *la_issued + 1;
    };
    // log alpha of chunk c (landed in P_LA) -> G in place, E_C, exact-path
    // flag; threads kScan0 .. kScan0 + 255: channel j, rows 32 rg .. 32 rg + 31
    auto scan_chunk = [&](int c) {
        const int t = tid - kG2cScan0, j = t & 127, rg = t >> 7;
        if (t == 0) {
            xflag[c & 1] = 0;
            if (!mbar_wait(tma_la, (uint32_t)(c & 1))) *abort_flag = 1;
            else *la_done = *la_done + 1;
        }
        asm volatile("barrier.sync 3, %0;" ::"n"(kG2cScanThreads) : "memory");
        if (*abort_flag) return;
        float g[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) g[i] = sg[(rg * 32 + i) * 128 + j];  // rows past T read as zero
#pragma unroll
        for (int i = 1; i < 32; ++i) g[i] += g[i - 1];
        scan[rg * 128 + j] = g[31];
        asm volatile("barrier.sync 3, %0;" ::"n"(kG2cScanThreads) : "memory");
        const float first = scan[j], tot = first + scan[128 + j];
        const float off = rg ? first : 0.f;
        if (rg == 0) {
            ec_of(c)[j] = expf(tot);
            if (-tot > 80.f) xflag[c & 1] = 1;
        }
#pragma unroll
        for (int i = 0; i < 32; ++i) sg[(rg * 32 + i) * 128 + j] = g[i] + off;
    };

    uint32_t mma_phase = 0;
    if (tid == 0) {
        issue_kq(0);
        if (nch > 1) issue_kq(1);
        issue_la(0);
    }
    __syncthreads();
    if (tid >= kG2cScan0) scan_chunk(0);
    __syncthreads();

#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        const int s = n & 1, cn = chunk_of(n);
        const int t0 = cn * kChunk, nv = min(kChunk, T - t0);
        const size_t tok0 = ((size_t)b * T + t0) * H + h;
        uint8_t *stg = sm + L::P_STG + s * L::H_TILES;
        const float *ec = ec_of(n);
        if (tid == 0 && !*abort_flag) {
            if (!mbar_wait(&tma_kq[s], (uint32_t)((n >> 1) & 1))) *abort_flag = 1;
            else kq_done[s] = kq_done[s] + 1;
        }
        __syncthreads();
        if (*abort_flag) break;
        const bool exact = xflag[s] != 0;

        // 1. operand tiles: thread items (row r, 8 channels) build 16 bytes of
        // every tile at the swizzled position of the TMA tile they come from.
        // b is read first: the tiles overwrite its pieces.
        float bq[2][8];
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int item = tid + m * kG2Threads, r = item >> 4, c8 = (item & 15) * 8;
            const uint32_t piece = r < 32 ? (uint32_t)(r >> 4) * 16384 : L::H_TB + (uint32_t)((r >> 4) - 2) * 8192;
            load8(reinterpret_cast<const float *>(stg + piece + (r & 15) * 512) + c8, bq[m]);
        }
        __syncthreads();
        {
            float ecv[8];
            load8(ec + (tid & 15) * 8, ecv);
#pragma unroll
            for (int m = 0; m < 2; ++m) {
                const int item = tid + m * kG2Threads, r = item >> 4, c8 = (item & 15) * 8;
                const int hj = c8 >> 6;
                const uint32_t off = sw128_offset(r, (c8 & 63) >> 3);
                uint8_t *kt = stg + L::H_KTL + hj * 8192 + off, *qt = stg + L::H_KQE + hj * 16384 + 8192 + off;
                float G[8], kk[8], qq[8];
                load8(sg + r * 128 + c8, G);
                load8(reinterpret_cast<const __nv_bfloat16 *>(kt), kk);
                load8(reinterpret_cast<const __nv_bfloat16 *>(qt), qq);
                float kbe[8], qe[8], kie[8], ktl[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float e = __expf(G[i]);
                    kbe[i] = kk[i] * bq[m][i] * e;
                    qe[i] = qq[i] * e;
                    kie[i] = -G[i] <= 80.f ? __fdividef(kk[i], e) : 0.f;
                }
                if (!exact) {  // K exp(G_C - G) = (K/E) exp(G_C), with E_C = exp(G_C) <= 1
#pragma unroll
                    for (int i = 0; i < 8; ++i) ktl[i] = kie[i] * ecv[i];
                } else {
                    float Gc[8];
                    load8(sg + 63 * 128 + c8, Gc);
#pragma unroll
                    for (int i = 0; i < 8; ++i) ktl[i] = kk[i] * __expf(Gc[i] - G[i]);
                }
                st_bf16x8(stg + L::H_KQE + hj * 16384 + off, kbe);
                st_bf16x8(qt, qe);
                st_bf16x8(stg + L::H_TB + hj * 8192 + off, kie);
                st_bf16x8(kt, ktl);
            }
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // 2. [K*B*E; Q*E] (K/E)^T -> A (lanes 0-63), P (lanes 64-127).  Meanwhile
        // the loader thread issues log alpha of chunk n+1 (G is consumed unless
        // the exact path reads it) and, once the copy of chunk n-1 out of the
        // other slot has landed, that slot's raw K/Q and b (chunk 1's went out
        // up front).
        if (tid == 0) {
            tc_after_sync();
            const uint32_t kqe = sbase + L::P_STG + s * L::H_TILES + L::H_KQE;
            const uint32_t kie = sbase + L::P_STG + s * L::H_TILES + L::H_TB;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem, smem_desc_sw128(kqe + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(kie + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
            mma_commit(mma_bar);
            if (!mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
        } else if (tid == kG2cLoader) {
            if (!exact && n + 1 < nch) issue_la(n + 1);
            if (n >= 1 && n + 1 < nch) {
                if (!mbar_wait(&landed[s ^ 1], (uint32_t)(((n - 1) >> 1) & 1))) *abort_flag = 1;
                else issue_kq(n + 1);
            }
        }
        mma_phase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        // K/E has been read: T's tile is cleared (the inverse writes only its lower triangle)
        *reinterpret_cast<uint4 *>(stg + L::H_TB + tid * 16) = make_uint4(0, 0, 0, 0);
        float *tp = TP_chunks ? TP_chunks + ((size_t)bh * nch + cn) * 2 * kChunk * kChunk : nullptr;
        if (!exact) {
            float v[16];
            tmem_ld16(tl + wc * 16, v);
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
                for (int ch = 0; ch < 2; ++ch) st_bf16x8(stg + L::H_PB + sw128_offset(r, wc * 2 + ch), v + 8 * ch);
                if (tp) {  // P in fp32 for the backward (second 64 x 64 block of the chunk)
                    float4 *dst = reinterpret_cast<float4 *>(tp + kChunk * kChunk + r * kChunk + i0);
#pragma unroll
                    for (int k4 = 0; k4 < 4; ++k4)
                        dst[k4] = make_float4(v[4 * k4], v[4 * k4 + 1], v[4 * k4 + 2], v[4 * k4 + 3]);
                }
            }
        } else {
            // some channel decays past e^80 in this chunk: A and P term by term
            // (pairs p = tid + 512 m), from k, q and b in global memory
#pragma unroll 1
            for (int m = 0; m < 8; ++m) {
                const int p = tid + m * kG2Threads, r = p >> 6, i = p & 63;
                float a = 0.f, pq = 0.f;
                if (i <= r && r < nv) {
                    const __nv_bfloat16 *kr = kg + (tok0 + (size_t)r * H) * D, *ki = kg + (tok0 + (size_t)i * H) * D;
                    const __nv_bfloat16 *qr = qg + (tok0 + (size_t)r * H) * D;
                    const float *br = bgate + (tok0 + (size_t)r * H) * D;
                    for (int jj = 0; jj < D; ++jj) {
                        const float kij = __bfloat162float(ki[jj]) * __expf(sg[r * D + jj] - sg[i * D + jj]);
                        pq = fmaf(__bfloat162float(qr[jj]), kij, pq);
                        if (i < r) a = fmaf(__bfloat162float(kr[jj]) * br[jj], kij, a);
                    }
                }
                sA[r * kLdT + i] = a;
                st_sw_bf16(stg + L::H_PB, r, i, pq);
                if (tp) tp[kChunk * kChunk + p] = pq;
            }
            __syncthreads();  // G is consumed
            if (tid == 0 && n + 1 < nch) issue_la(n + 1);
        }
        __syncthreads();

        // 3. inverse (warps 0 and 1; T also in bf16 into the staging slot)
        // while warps 8-15 scan log alpha of chunk n+1
        if (warp < 2) inverse_two_warps(sA, sT, warp, lane, 1, TEmit{stg + L::H_TB, nullptr, ones, ones});
        else if (tid >= kG2cScan0 && n + 1 < nch) scan_chunk(n + 1);
        __syncthreads();
        if (tp) {  // T in fp32 for the backward (its upper triangle as zeros)
            for (int idx = tid; idx < kChunk * kChunk; idx += kG2Threads) {
                const int r = idx >> 6, i = idx & 63;
                tp[idx] = i <= r ? sT[r * kLdT + i] : 0.f;
            }
        }
        fence_async_smem();
        __syncthreads();
        // 4. the tiles and E_C into the state CTA's slot s, once the state CTA
        // has finished chunk n-2 there
        if (tid == 0 && !*abort_flag) {
            if (n >= 2 && !mbar_wait(&empty[s], (uint32_t)(((n >> 1) - 1) & 1))) *abort_flag = 1;
            else {
                bulk_copy_to_cluster(remote_slot0 + s * L::H_TILES, stg, L::H_TILES, remote_full0 + 8 * s);
                bulk_copy_to_cluster(remote_ec0 + s * L::H_EC, ec, L::H_EC, remote_full0 + 8 * s);
            }
        }
    }

    __syncthreads();
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        // drain: every TMA load still in flight, then the MMAs
        for (int sl = 0; sl < 2; ++sl)
            for (int k2 = kq_done[sl]; k2 < kq_issued[sl]; ++k2) mbar_wait(&tma_kq[sl], (uint32_t)(k2 & 1));
        for (int k2 = *la_done; k2 < *la_issued; ++k2) mbar_wait(tma_la, (uint32_t)(k2 & 1));
        mma_commit(mma_bar);
        mbar_wait(mma_bar, mma_phase);
    }
    tc_before_sync();
    __syncthreads();
    cluster_sync();  // the state CTA has received every copy and sent its last arrive
    if (warp == 0) {
        tc_after_sync();
        tmem_dealloc(tmem, 64);
    }
}

// ----------------------------------------------------------------- state CTA --
// Barriers (S_BAR): tma_full (V), hand_full[2] (filled by the prep's copies),
// a (the chunk's MMAs), b (W^T and U^gT of the next chunk); then the TMEM
// address and the abort flag.
__device__ __forceinline__ void g2c_state(uint8_t *sm, const CUtensorMap *tm_v, const CUtensorMap *tm_o, int T,
                                          int H, int b, int h, const float *wgate, const float *S0, float *S_T,
                                          bool store_o, float *S_chunks) {
    using L = G2cLayout;
    using namespace sm100;
    constexpr int D = 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;           // TMEM lane = row of S / U^T / O^T / W^T
    const int bh = b * H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *tma_full = reinterpret_cast<uint64_t *>(sm + L::S_BAR);
    uint64_t *hand_full = tma_full + 1;  // [2]
    uint64_t *bar_a = tma_full + 3, *bar_b = tma_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t sbase = smem_u32(sm);

    if (tid == 0) {
        mbar_init(tma_full, 1);
        mbar_init(&hand_full[0], 1);
        mbar_init(&hand_full[1], 1);
        mbar_init(bar_a, 1);
        mbar_init(bar_b, 1);
        fence_mbar_init();
        *abort_flag = 0;
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
    const uint32_t remote_empty0 = cluster_addr(sm + L::P_BAR + 8 * kG2cBarEmpty, 0);    // prep's empty[0]
    const uint32_t remote_landed0 = cluster_addr(sm + L::P_BAR + 8 * kG2cBarLanded, 0);  // prep's landed[0]

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
        tmem_st32(tl + kG2cS + col, v);
        tmem_wait_st();
    }

    int v_issued = 0, v_done = 0;  // V loads (thread 0's count)
    auto issue_tma_v = [&](int n) {
        mbar_expect_tx(tma_full, 16384);
#pragma unroll
        for (int half = 0; half < 2; ++half)
            tma_load_4d(sm + L::S_V + half * 8192, tm_v, tma_full, half * 64, h, n * kChunk, b);
        ++v_issued;
    };
    // W_gate*V of chunk n -> S_WV[n & 1] (every thread; the V tile has landed)
    auto build_wv = [&](int n) {
        const int t0 = n * kChunk, nv = min(kChunk, T - t0);
        const size_t tok0 = ((size_t)b * T + t0) * H + h;
        uint8_t *wv = sm + L::S_WV + (n & 1) * 16384;
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            const int item = tid + m * kG2Threads, r = item >> 4, c8 = (item & 15) * 8;
            const int hj = c8 >> 6;
            const uint32_t off = sw128_offset(r, (c8 & 63) >> 3);
            const size_t e = (tok0 + (size_t)r * H) * 128 + c8;
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            const float4 w0 = r < nv ? *reinterpret_cast<const float4 *>(wgate + e) : z;
            const float4 w1 = r < nv ? *reinterpret_cast<const float4 *>(wgate + e + 4) : z;
            const float ww[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            float vv[8];
            load8(reinterpret_cast<const __nv_bfloat16 *>(sm + L::S_V + hj * 8192 + off), vv);
#pragma unroll
            for (int i = 0; i < 8; ++i) vv[i] *= ww[i];
            st_bf16x8(wv + hj * 8192 + off, vv);
        }
        if (n + 1 < nch) {  // the next chunk's w gate rows -> L2
            const int nv1 = min(kChunk, T - t0 - kChunk);
            for (int k = tid; k < 64 * 4; k += kG2Threads) {
                const int r = k >> 2, line = k & 3;
                if (r < nv1) prefetch_l2(wgate + (tok0 + (size_t)(kChunk + r) * H) * 128 + line * 32);
            }
        }
    };
    // W^T = (K*B*E)^T T^T and U^gT = (W_gate*V)^T T^T of chunk n (thread 0), once its slot landed
    auto issue_wu = [&](int n) -> bool {
        const int s = n & 1;
        if (!mbar_wait_cluster(&hand_full[s], (uint32_t)((n >> 1) & 1))) return false;
        if (n + 2 < nch) mbar_arrive_remote(remote_landed0 + 8 * s);  // the prep may restage its slot
        tc_after_sync();
        const uint32_t hs = sbase + L::S_H + s * L::H_TILES, wv = sbase + L::S_WV + s * 16384;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kG2cW, smem_desc_sw128(hs + L::H_KQE + kk * 2048, 16384, 1024),
                     smem_desc_sw128(hs + L::H_TB + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kG2cU + 64 * s, smem_desc_sw128(wv + kk * 2048, 8192, 1024),
                     smem_desc_sw128(hs + L::H_TB + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
        mma_commit(bar_b);
        return true;
    };
    // W^T of chunk n (lane j, column r) -> W [j][r] bf16 over that slot's K*B*E,
    // the MN-major B operand of U^T -= S W^T (j-blocks of 64 rows 16 KB apart)
    auto convert_w = [&](int n) {
        float v[16];
        tmem_ld16(tl + kG2cW + wc * 16, v);
        uint8_t *wdst = sm + L::S_H + (n & 1) * L::H_TILES + L::H_KQE + (row >> 6) * 16384;
#pragma unroll
        for (int ch = 0; ch < 2; ++ch) st_bf16x8(wdst + sw128_offset(row & 63, wc * 2 + ch), v + 8 * ch);
        fence_async_smem();
    };
    // O^T of chunk n (lane = value channel, column = token) -> bf16 tile [token][channel]
    auto stage_o = [&](int n) {
        float v[16];
        tmem_ld16(tl + kG2cO + 64 * (n & 1) + wc * 16, v);
        uint8_t *half = sm + L::S_OST + (row >> 6) * 8192;
        const int cc = row & 63;
#pragma unroll
        for (int i = 0; i < 16; ++i) st_sw_bf16(half, wc * 16 + i, cc, v[i]);
        fence_async_smem();
    };
    auto store_o_tile = [&](int n) {  // thread 0, after a barrier that follows stage_o
        tma_store_4d(tm_o, sm + L::S_OST, 0, h, n * kChunk, b);
        tma_store_4d(tm_o, sm + L::S_OST + 8192, 64, h, n * kChunk, b);
        bulk_commit();
    };

    uint32_t aphase = 0, bphase = 0;
    // chunk 0's W_gate*V, W and U^g
    if (tid == 0) issue_tma_v(0);
    if (!mbar_wait(tma_full, 0)) *abort_flag = 1;
    else build_wv(0);
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    if (tid == 0) {
        if (!*abort_flag) {
            ++v_done;
            if (nch > 1) issue_tma_v(1);
            if (!issue_wu(0) || !mbar_wait(bar_b, bphase)) *abort_flag = 1;
        }
    }
    bphase ^= 1;
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    if (!*abort_flag) convert_w(0);
    tc_before_sync();
    __syncthreads();

    int n_done = 0;  // chunks whose MMAs all completed
#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        if (*abort_flag) break;
        const int s = n & 1;
        const uint32_t hs = sbase + L::S_H + s * L::H_TILES;
        const float *ecs = reinterpret_cast<const float *>(sm + L::S_EC + s * L::H_EC);
        const uint32_t uw = sbase + L::S_WV + s * 16384;

        // (a) S -> bf16 operand (and the fp32 entry state, when kept); S <- S Diag(E_C)
        {
            const int col = wc * 32;
            float v[32];
            tmem_ld32(tl + kG2cS + col, v);
            if (S_chunks) {
                float4 *dst = reinterpret_cast<float4 *>(S_chunks + (((size_t)bh * nch + n) * D + row) * D + col);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            uint8_t *half = sm + L::S_SB + (wc >> 1) * 16384;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) st_bf16x8(half + sw128_offset(row, (wc & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= ecs[col + i];
            tmem_st32(tl + kG2cS + col, v);
            tmem_wait_st();
        }
        fence_async_smem();
        if (tid == 0) bulk_wait_read_all();  // the O tile of chunk n-2 has left shared memory
        tc_before_sync();
        __syncthreads();

        // (b) U^T -= S W^T ; O^T = S (Q*E)^T
        if (tid == 0) {
            tc_after_sync();
            const uint32_t sb = sbase + L::S_SB;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2cU + 64 * s, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(hs + L::H_KQE + (kk >> 2) * 16384 + (kk & 3) * 2048, 8192, 1024),
                         idesc_bf16(128, 64, false, true, true), 1);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2cO + 64 * s, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(hs + L::H_KQE + 8192 + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
            mma_commit(bar_a);
        }
        __syncwarp();
        // (c) stage the previous chunk's output; the next chunk's W_gate*V, then its W and U^g
        if (store_o && n > 0) stage_o(n - 1);
        if (n + 1 < nch) {
            if (!mbar_wait(tma_full, (uint32_t)((n + 1) & 1))) *abort_flag = 1;
            else build_wv(n + 1);
            fence_async_smem();
            tc_before_sync();
            __syncthreads();
            if (tid == 0 && !*abort_flag) {
                ++v_done;
                if (n + 2 < nch) issue_tma_v(n + 2);  // the V tile is consumed
                if (!issue_wu(n + 1)) *abort_flag = 1;
            }
        }
        // (d) U^T -> bf16 A operand over this chunk's W_gate*V
        if (tid == 0 && !mbar_wait(bar_a, aphase)) *abort_flag = 1;
        aphase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        if (tid == 0 && store_o && n > 0) store_o_tile(n - 1);
        {
            float v[16];
            tmem_ld16(tl + kG2cU + 64 * s + wc * 16, v);
#pragma unroll
            for (int ch = 0; ch < 2; ++ch)
                st_bf16x8(sm + L::S_WV + s * 16384 + sw128_offset(row, wc * 2 + ch), v + 8 * ch);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // (e) O^T += U^T P^T ; S += U^T (K * exp(G_C - G))
        if (tid == 0) {
            tc_after_sync();
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2cO + 64 * s, smem_desc_sw128(uw + kk * 32, 16, 1024),
                         smem_desc_sw128(hs + L::H_PB + kk * 32, 16, 1024), idesc_bf16(128, 64, false, false), 1);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2cS, smem_desc_sw128(uw + kk * 32, 16, 1024),
                         smem_desc_sw128(hs + L::H_KTL + kk * 2048, 8192, 1024), idesc_bf16(128, 128, false, true),
                         1);
            mma_commit(bar_a);
            if (n + 1 < nch && !mbar_wait(bar_b, bphase)) *abort_flag = 1;
        }
        if (n + 1 < nch) bphase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        // (f) W of the next chunk over its slot's K*B*E (its MMAs are done)
        if (n + 1 < nch) convert_w(n + 1);
        // (g) chunk n finished: give its slot back to the prep CTA
        if (tid == 0) {
            if (!mbar_wait(bar_a, aphase)) *abort_flag = 1;
            else {
                n_done = n + 1;
                if (n + 2 < nch) {
                    mbar_expect_tx(&hand_full[s], L::H_BYTES);
                    mbar_arrive_remote(remote_empty0 + 8 * s);
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
            const int col = wc * 32;
            tmem_ld32(tl + kG2cS + col, v);
            float4 *dst = reinterpret_cast<float4 *>(S_T + ((size_t)bh * D + row) * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
    }
    if (tid == 0) bulk_wait_all();  // output stores complete before the CTA exits
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        // drain: this CTA's V loads, its MMAs, and the prep CTA's copies into it
        for (int k2 = v_done; k2 < v_issued; ++k2) mbar_wait(tma_full, (uint32_t)(k2 & 1));
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

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kG2Threads, 1)
gdr2_fwd_tc2_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                    const __grid_constant__ CUtensorMap tm_v, const __grid_constant__ CUtensorMap tm_o,
                    const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_bg,
                    const __nv_bfloat16 *__restrict__ kg, const __nv_bfloat16 *__restrict__ qg,
                    int T, int H, const float *__restrict__ bgate,
                    const float *__restrict__ wgate, const float *__restrict__ S0, float *__restrict__ S_T,
                    int store_o, float *__restrict__ S_chunks, float *__restrict__ TP_chunks) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int bh = blockIdx.x >> 1, b = bh / H, h = bh % H;
    if (sm100::cluster_ctarank() == 0)
        g2c_prep(sm, &tm_q, &tm_k, &tm_la, &tm_bg, T, H, b, h, kg, qg, bgate, TP_chunks);
    else
        g2c_state(sm, &tm_v, &tm_o, T, H, b, h, wgate, S0, S_T, store_o != 0, S_chunks);
}

// 4-D map over a [B, T, H, d] fp32 gate tensor: box = d channels x 1 head x
// `rows` tokens x 1 batch, rows of d floats unswizzled; tokens past T read as zero.
inline bool make_gate_map(CUtensorMap *map, const float *base, int B, int T, int H, int d, int rows = kChunk) {
    EncodeTiledFn enc = encode_tiled_fn();
    if (!enc) return false;
    const cuuint64_t dims[4] = {(cuuint64_t)d, (cuuint64_t)H, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[3] = {(cuuint64_t)d * 4, (cuuint64_t)H * d * 4, (cuuint64_t)T * H * d * 4};
    const cuuint32_t box[4] = {(cuuint32_t)d, 1, (cuuint32_t)rows, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, const_cast<float *>(base), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Same arguments and outputs as launch_fwd2_tc (fwd2_tc.cuh).
inline cudaError_t launch_fwd2_tc2(int B, int T, int H, const void *q, const void *k, const void *v,
                                   const float *la, const float *bgate, const float *wgate, const float *S0,
                                   void *o, float *S_T, cudaStream_t stream, float *S_chunks = nullptr,
                                   float *TP_chunks = nullptr) {
    CUtensorMap mq, mk, mv, mo, mla, mbg;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128) || !make_token_map(&mo, o ? o : q, B, T, H, 128) ||
        !make_gate_map(&mla, la, B, T, H, 128) || !make_gate_map(&mbg, bgate, B, T, H, 128, 16))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr2_fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)G2cLayout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr2_fwd_tc2_kernel<<<(unsigned)(2 * B * H), kG2Threads, G2cLayout::kAlloc, stream>>>(
        mq, mk, mv, mo, mla, mbg, static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(q), T, H,
        bgate, wgate, S0, S_T, o != nullptr ? 1 : 0, S_chunks, TP_chunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
