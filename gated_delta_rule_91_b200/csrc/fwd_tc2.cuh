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
// four); one thread per CTA issues TMA and MMA.  Sixteen warps (four per SM
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
    static constexpr uint32_t P_STG = P_T + 64 * kLdT * 4;  // 3 staging slots
    static constexpr uint32_t P_GATE = P_STG + 3 * H_SLOT;  // 2 x {g, beta, gamma, dec, gamma', 1/gamma' [64], flag}
    static constexpr uint32_t P_GATE_BYTES = 6 * 256 + 16;
    static constexpr uint32_t P_BAR = P_GATE + 2 * P_GATE_BYTES;
    static constexpr uint32_t P_BYTES = P_BAR + 128;
    static constexpr uint32_t kAlloc = (S_BYTES > P_BYTES ? S_BYTES : P_BYTES) + 1024;
};
static_assert(Tc2Layout::S_H % 1024 == 0 && Tc2Layout::S_W % 1024 == 0 && Tc2Layout::S_SB % 1024 == 0 &&
                  Tc2Layout::S_OST % 1024 == 0,
              "state tiles must be 1024-aligned");
static_assert(Tc2Layout::P_STG % 1024 == 0 && Tc2Layout::H_SLOT % 1024 == 0, "slots must be 1024-aligned");
static_assert(Tc2Layout::kAlloc <= 232448, "shared memory budget");
static_assert(Tc2Layout::H_T2 == Tc2Layout::H_T1 + 8192, "T' and T'' are adjacent");

// state TMEM columns (512 allocated)
constexpr uint32_t kT2S = 0, kT2W = 128, kT2U = 192, kT2O = 320;  // U, O double-buffered (+64)

// T = (I + A)^{-1} for strictly lower 64 x 64 A (fp32, row stride kLdT) by
// recursive doubling over 16 x 16 blocks, solved by two warps:
//   diagonal blocks t_0..t_3 by substitution (lane j owns column j of one
//   block; each warp takes two blocks);
//   32 level, block P (o = 32P, one warp each):
//     T[o+16:o+32, o:o+16] = -t_{2P+1} (A[o+16:o+32, o:o+16] t_{2P});
//   64 level, in 8-column slabs (two per warp):
//     T[32:64, 0:32] = -T22 (A[32:64, 0:32] T11).
// Products run on warp-level tensor-core tiles (m16n8k8, tf32 operands,
// fp32 accumulation); the known zero blocks of T11 and T22 are skipped.  Intermediate products are parked in A's unused upper
// triangle; only the lower triangle of T is written.
// Optional bf16 copies of T with scaled columns, written as the blocks of T are
// produced: t1 = T diag(beta), t2 = T diag(beta gamma), 128B-swizzled [r][i]
// tiles; only the lower triangle (diagonal blocks whole) is written.
struct TEmit {
    uint8_t *t1, *t2;           // t1 nullptr: no copies; t2 nullptr: t1 only
    const float *beta, *gamma;  // [64]
};

__device__ __forceinline__ void inverse_diag16(const float *sA, float *sT, int blk, int j, const TEmit &em) {
    constexpr int LD = kLdT;
    const int base = blk * 16;
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
    if (em.t1) {
        const int c = base + j;
        const float b1 = em.beta[c], b2 = b1 * em.gamma[c];
#pragma unroll
        for (int r = 0; r < 16; ++r) {
            sm100::st_sw_bf16(em.t1, base + r, c, t[r] * b1);
            if (em.t2) sm100::st_sw_bf16(em.t2, base + r, c, t[r] * b2);
        }
    }
}

__device__ __forceinline__ uint32_t to_tf32(float x) {
    uint32_t r;
    asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(r) : "f"(x));
    return r;
}
__device__ __forceinline__ void mma_tf32_16x8x8(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k8.row.col.f32.tf32.tf32.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// acc[m][n] (16 x 8 tiles) += A (16*MT x 8*NK8, from Ab) * B (8*NK8 x 8*NT,
// from Bb); both fp32 row-major with stride kLdT.  Tile (m, k) is skipped
// when k >= kmax[m] (a known zero block of A).  Fragment ownership (lane =
// 4g + t): A rows g, g+8 and columns t, t+4; B rows t, t+4 and column g; acc
// rows g, g+8 and columns 2t, 2t+1.  With kInverseSplitTf32 each operand is
// split into tf32 hi + lo and the product keeps hi*hi + hi*lo + lo*hi.
constexpr bool kInverseSplitTf32 = false;
template <int MT, int NT, int NK8>
__device__ __forceinline__ void warp_mm(float (&acc)[MT][NT][4], const float *Ab, const float *Bb,
                                        const int (&kmax)[MT], int lane) {
    constexpr int LD = kLdT;
    const int g = lane >> 2, t = lane & 3;
#pragma unroll
    for (int kk = 0; kk < NK8; ++kk) {
        uint32_t ah[MT][4], al[MT][4], bh[NT][2], bl[NT][2];
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            const float *ap = Ab + m * 16 * LD + kk * 8;
            const float av[4] = {ap[g * LD + t], ap[(g + 8) * LD + t], ap[g * LD + t + 4], ap[(g + 8) * LD + t + 4]};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                ah[m][i] = to_tf32(av[i]);
                al[m][i] = kInverseSplitTf32 ? to_tf32(av[i] - __uint_as_float(ah[m][i])) : 0u;
            }
        }
#pragma unroll
        for (int n = 0; n < NT; ++n) {
            const float *bp = Bb + kk * 8 * LD + n * 8;
            const float bv[2] = {bp[t * LD + g], bp[(t + 4) * LD + g]};
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                bh[n][i] = to_tf32(bv[i]);
                bl[n][i] = kInverseSplitTf32 ? to_tf32(bv[i] - __uint_as_float(bh[n][i])) : 0u;
            }
        }
#pragma unroll
        for (int m = 0; m < MT; ++m) {
            if (kk >= kmax[m]) continue;
#pragma unroll
            for (int n = 0; n < NT; ++n) {
                if (kInverseSplitTf32) {
                    mma_tf32_16x8x8(acc[m][n], al[m], bh[n][0], bh[n][1]);
                    mma_tf32_16x8x8(acc[m][n], ah[m], bl[n][0], bl[n][1]);
                }
                mma_tf32_16x8x8(acc[m][n], ah[m], bh[n][0], bh[n][1]);
            }
        }
    }
}
__device__ __forceinline__ void warp_store16x8(float *Db, const float (&acc)[4], float scale, int lane) {
    constexpr int LD = kLdT;
    const int g = lane >> 2, t = lane & 3;
    *reinterpret_cast<float2 *>(Db + g * LD + 2 * t) = make_float2(scale * acc[0], scale * acc[1]);
    *reinterpret_cast<float2 *>(Db + (g + 8) * LD + 2 * t) = make_float2(scale * acc[2], scale * acc[3]);
}

// The bf16 copies of one 16 x 8 fragment of T (scaled by `scale`) at (row0, col0).
__device__ __forceinline__ void emit16x8(const TEmit &em, int row0, int col0, const float (&acc)[4], float scale,
                                         int lane) {
    const int g = lane >> 2, c = col0 + 2 * (lane & 3);
    const float ba = scale * em.beta[c], bb = scale * em.beta[c + 1];
    const float ga = ba * em.gamma[c], gb = bb * em.gamma[c + 1];
    sm100::st_sw_bf16x2(em.t1, row0 + g, c, acc[0] * ba, acc[1] * bb);
    sm100::st_sw_bf16x2(em.t1, row0 + g + 8, c, acc[2] * ba, acc[3] * bb);
    if (em.t2) {
        sm100::st_sw_bf16x2(em.t2, row0 + g, c, acc[0] * ga, acc[1] * gb);
        sm100::st_sw_bf16x2(em.t2, row0 + g + 8, c, acc[2] * ga, acc[3] * gb);
    }
}

// The whole inverse, run by the two warps w = 0, 1 of the calling CTA;
// `bar_id` names a 64-thread barrier between the 32 and 64 levels.
__device__ __forceinline__ void inverse_two_warps(float *sA, float *sT, int w, int lane, int bar_id,
                                                  const TEmit &em) {
    constexpr int LD = kLdT;
    inverse_diag16(sA, sT, 2 * w + (lane >> 4), lane & 15, em);
    __syncwarp();
    {   // 32 level, block P = w
        const int o = 32 * w;
        const int k2[1] = {2};
        float acc[1][2][4] = {};
        // X = A[o+16:o+32, o:o+16] t_{2P} -> parked in A[o:o+16, o+16:o+32]
        warp_mm<1, 2, 2>(acc, sA + (o + 16) * LD + o, sT + o * LD + o, k2, lane);
        warp_store16x8(sA + o * LD + o + 16, acc[0][0], 1.f, lane);
        warp_store16x8(sA + o * LD + o + 24, acc[0][1], 1.f, lane);
        __syncwarp();
        float acc2[1][2][4] = {};
        // T[o+16:o+32, o:o+16] = -t_{2P+1} X
        warp_mm<1, 2, 2>(acc2, sT + (o + 16) * LD + o + 16, sA + o * LD + o + 16, k2, lane);
        warp_store16x8(sT + (o + 16) * LD + o, acc2[0][0], -1.f, lane);
        warp_store16x8(sT + (o + 16) * LD + o + 8, acc2[0][1], -1.f, lane);
        if (em.t1) {
            emit16x8(em, o + 16, o, acc2[0][0], -1.f, lane);
            emit16x8(em, o + 16, o + 8, acc2[0][1], -1.f, lane);
        }
    }
    asm volatile("barrier.sync %0, 64;" ::"r"(bar_id) : "memory");
    {   // 64 level: slabs c0 = 8w (T11 rows 0:32) and 16 + 8w (T11 rows 16:32 only)
        const int c0 = 8 * w, c1 = 16 + 8 * w;
        const int k4[2] = {4, 4}, k2[2] = {2, 2};
        float x0[2][1][4] = {}, x1[2][1][4] = {};
        // X = A[32:64, 0:32] T11[:, slab] -> parked in A[0:32, 32 + slab]
        warp_mm<2, 1, 4>(x0, sA + 32 * LD, sT + c0, k4, lane);
        warp_mm<2, 1, 2>(x1, sA + 32 * LD + 16, sT + 16 * LD + c1, k2, lane);
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            warp_store16x8(sA + 16 * m * LD + 32 + c0, x0[m][0], 1.f, lane);
            warp_store16x8(sA + 16 * m * LD + 32 + c1, x1[m][0], 1.f, lane);
        }
        __syncwarp();
        // T[32:64, slab] = -T22 X  (T22[0:16, 16:32] = 0)
        const int kt[2] = {2, 4};
        float y0[2][1][4] = {}, y1[2][1][4] = {};
        warp_mm<2, 1, 4>(y0, sT + 32 * LD + 32, sA + 32 + c0, kt, lane);
        warp_mm<2, 1, 4>(y1, sT + 32 * LD + 32, sA + 32 + c1, kt, lane);
#pragma unroll
        for (int m = 0; m < 2; ++m) {
            warp_store16x8(sT + (32 + 16 * m) * LD + c0, y0[m][0], -1.f, lane);
            warp_store16x8(sT + (32 + 16 * m) * LD + c1, y1[m][0], -1.f, lane);
            if (em.t1) {
                emit16x8(em, 32 + 16 * m, c0, y0[m][0], -1.f, lane);
                emit16x8(em, 32 + 16 * m, c1, y1[m][0], -1.f, lane);
            }
        }
    }
}

// ------------------------------------------------------------------ prep CTA --
// Prep-CTA roles: warps 0 and 1 (which hold only rows of A in the mask step)
// solve the inverse while the other fourteen warps stage P, Q~ and the gates
// into a local slot and warp 8 computes the next chunk's gates; lane 0 of the
// last warp issues TMA, MMA and the bulk copy.  Three local staging slots feed the state CTA's two: the
// local slot of chunk n was last read by the copy of chunk n-3, which the
// state CTA confirmed before chunk n-1 went out, so staging never waits; only
// the copy waits for the state CTA's slot.
constexpr int kPrepIssuer = kTc2Threads - 32;
constexpr int kPrepGateWarp = 8;
constexpr int kPrepStagers = kTc2Threads - 2 * 32;  // warps 2-15 (named barrier 1)
constexpr int kPrepQtStagers = kPrepStagers - 32;  // the issuer's warp skips the Q~ copy
constexpr int kPrepSolverBarrier = 2;               // the two solver warps

// `reverse` walks the chunks from last to first (the backward's dS pass):
// step n then works on chunk nch-1-n; everything else is unchanged.
__device__ __forceinline__ void tc2_prep(uint8_t *sm, const CUtensorMap *tm_q, const CUtensorMap *tm_k,
                                         int T, int H, int b, int h, const float *log_alpha,
                                         const float *beta, bool reverse = false) {
    using L = Tc2Layout;
    using namespace sm100;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int nch = (T + kChunk - 1) / kChunk;
    const bool issuer = tid == kPrepIssuer;
    const bool solver = warp < 2;
    const int srank = tid - 64;  // rank among the staging warps
    uint64_t *tma_full = reinterpret_cast<uint64_t *>(sm + L::P_BAR);  // [2]
    uint64_t *empty = tma_full + 2;                                      // [2], arrived by the state CTA
    uint64_t *mma_bar = tma_full + 4;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(tma_full + 5);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    float *sA = reinterpret_cast<float *>(sm + L::P_A), *sT = reinterpret_cast<float *>(sm + L::P_T);
    const uint32_t sbase = smem_u32(sm);
    // gate arrays of chunk parity `par`: g, beta, gamma, dec, gamma', 1/gamma', exact flag
    auto gates_of = [&](int par) { return reinterpret_cast<float *>(sm + L::P_GATE + par * L::P_GATE_BYTES); };

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
    // T' and T'' of every staging slot: zero once; the inverse writes only the
    // lower triangle, so the upper blocks stay zero
    for (int k = tid; k < 3 * 1024; k += kTc2Threads) {
        const int slot = k >> 10, off = (k & 1023) * 16;  // H_T1 and H_T2 are adjacent (16 KB)
        *reinterpret_cast<uint4 *>(sm + L::P_STG + slot * L::H_SLOT + L::H_T1 + off) = make_uint4(0, 0, 0, 0);
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
        const int c = reverse ? nch - 1 - n : n;
        mbar_expect_tx(&tma_full[s], 32768);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
            tma_load_4d(kq + half * 16384, tm_k, &tma_full[s], half * 64, h, c * kChunk, b);
            tma_load_4d(kq + half * 16384 + 8192, tm_q, &tma_full[s], half * 64, h, c * kChunk, b);
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
    // gates of one chunk, held by the gate warp (lane l: rows 2l, 2l+1) between load and use
    float pl0 = 0.f, pl1 = 0.f, pb0 = 0.f, pb1 = 0.f;
    auto load_gates = [&](int n) {
        const int c0 = (reverse ? nch - 1 - n : n) * kChunk, nv = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        const int r0 = 2 * lane, r1 = r0 + 1;
        pl0 = r0 < nv ? log_alpha[tok0 + (size_t)r0 * H] : 0.f;
        pl1 = r1 < nv ? log_alpha[tok0 + (size_t)r1 * H] : 0.f;
        pb0 = r0 < nv ? beta[tok0 + (size_t)r0 * H] : 0.f;
        pb1 = r1 < nv ? beta[tok0 + (size_t)r1 * H] : 0.f;
    };
    // g (inclusive prefix sum), gamma, dec, gamma' = exp(g - g_31), 1/gamma', exact flag
    auto compute_gates = [&](float *G) {
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
        G[r0] = g0; G[r1] = g1;
        G[64 + r0] = pb0; G[64 + r1] = pb1;
        G[128 + r0] = expf(g0); G[128 + r1] = expf(g1);
        G[192 + r0] = expf(gC - g0); G[192 + r1] = expf(gC - g1);
        G[256 + r0] = expf(g0 - gM); G[256 + r1] = expf(g1 - gM);
        G[320 + r0] = expf(gM - g0); G[320 + r1] = expf(gM - g1);
        if (lane == 0) reinterpret_cast<volatile int *>(G + 384)[0] = (gF - gC) > 80.f;
    };
    if (warp == kPrepGateWarp) {
        load_gates(0);
        compute_gates(gates_of(0));
        if (nch > 1) load_gates(1);  // prefetch: consumed during chunk 0
    }

    int tma_issued = 0, tma_done = 0;
    uint32_t mma_phase = 0;
    int ls = 0;  // local staging slot of chunk n (n mod 3)
    if (issuer) {
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
        uint8_t *stg = sm + L::P_STG + ls * L::H_SLOT;
        const float *G = gates_of(s);
        const float *sg = G, *sbeta = G + 64, *sgam = G + 128, *sdec = G + 192, *sgp = G + 256, *sinv = G + 320;
        __syncthreads();
        if (*abort_flag) break;
        if (issuer && !mbar_wait(mma_bar, mma_phase)) *abort_flag = 1;
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
            const bool exact = reinterpret_cast<const volatile int *>(G + 384)[0] != 0;
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

        if (solver) {
            inverse_two_warps(sA, sT, warp, lane, kPrepSolverBarrier,
                              TEmit{stg + L::H_T1, stg + L::H_T2, sbeta, sgam});
        } else {
            if (issuer && n + 1 < nch) {  // next chunk's K K^T / Q K^T overlaps this chunk's inverse
                tc_after_sync();
                if (!mbar_wait(&tma_full[s ^ 1], (uint32_t)(((n + 1) >> 1) & 1))) *abort_flag = 1;
                else {
                    ++tma_done;
                    issue_mma1(s ^ 1);
                }
            }
            float *hg = reinterpret_cast<float *>(stg + L::H_G);
            if (srank < 128) hg[srank] = srank < 64 ? sgam[srank] : sdec[srank - 64];
            if (row >= 64) {  // P rows
#pragma unroll
                for (int ch = 0; ch < 2; ++ch)
                    st_bf16x8(stg + L::H_P + sw128_offset(row - 64, wc * 2 + ch), pv + 8 * ch);
            }
            // Q~ = diag(gamma) Q: same swizzled positions as the Q tile
            const uint8_t *qt = sm + L::P_KQ + s * 32768 + 8192;
            if (srank < kPrepQtStagers) {
                for (int ci = srank; ci < 1024; ci += kPrepQtStagers) {  // 16-byte chunks
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
            asm volatile("barrier.sync 1, %0;" ::"n"(kPrepStagers) : "memory");
            if (issuer && n + 2 < nch && !*abort_flag) {  // K/Q stage s is free: MMA done, Q read
                issue_tma(n + 2, s);
                ++tma_issued;
            }
            if (warp == kPrepGateWarp && n + 1 < nch) {  // next chunk's gates (other buffer)
                compute_gates(gates_of(s ^ 1));
                if (n + 2 < nch) load_gates(n + 2);
            }
        }
        fence_async_smem();
        __syncthreads();
        if (*abort_flag) break;
        if (issuer) {
            // the state CTA's slot s must have been consumed (chunk n-2)
            if (n >= 2 && !mbar_wait_cluster(&empty[s], (uint32_t)(((n >> 1) - 1) & 1))) *abort_flag = 1;
            else bulk_copy_to_cluster(remote_slot0 + s * L::H_SLOT, stg, L::H_BYTES, remote_full0 + 8 * s);
        }
        ls = ls == 2 ? 0 : ls + 1;
    }

    if (*abort_flag && issuer) {
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
                                          const float *S0, float *S_T, bool store_o, uint8_t *S_tiles) {
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
            if (S_tiles) {  // the bf16 entry state of chunk n, as swizzled, for the backward
                bulk_store_s2g(S_tiles + ((size_t)bh * nch + n) * 32768, sm + L::S_SB, 32768);
                bulk_commit();
            }
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
        if (tid == 0 && S_tiles) bulk_wait_read_all();  // the state copy has left S_SB
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
                   uint8_t *__restrict__ S_tiles) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int bh = blockIdx.x >> 1, b = bh / H, h = bh % H;
    if (sm100::cluster_ctarank() == 0)
        tc2_prep(sm, &tm_q, &tm_k, T, H, b, h, log_alpha, beta);
    else
        tc2_state(sm, &tm_k, &tm_v, &tm_o, T, H, b, h, S0, S_T, store_o != 0, S_tiles);
}

// o == nullptr runs the recurrence without writing outputs (the backward's
// recompute); S_tiles (nullable) receives every chunk's entry state as the
// bf16 MMA operand tile, [B, H, nchunks] x 32 KB: two 64-column halves of
// [128 rows][64 columns], 128-byte rows, 128B-swizzled.
inline cudaError_t launch_fwd_tc2(int B, int T, int H, const void *q, const void *k, const void *v,
                                  const float *la, const float *beta, const float *S0, void *o,
                                  float *S_T, cudaStream_t stream, uint8_t *S_tiles = nullptr) {
    CUtensorMap mq, mk, mv, mo;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_token_map(&mv, v, B, T, H, 128) || !make_token_map(&mo, o ? o : q, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr_fwd_tc2_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)Tc2Layout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr_fwd_tc2_kernel<<<(unsigned)(2 * B * H), kTc2Threads, Tc2Layout::kAlloc, stream>>>(
        mq, mk, mv, mo, T, H, la, beta, S0, S_T, o != nullptr ? 1 : 0, S_tiles);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
