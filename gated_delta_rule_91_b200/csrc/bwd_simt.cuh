// bwd_simt.cuh -- chunkwise backward of the gated delta rule on CUDA cores
// (fp32 arithmetic, fp32 or bf16 inputs).
//
// The pages give no backward; this is the chain rule applied to the chunk
// map of the forward (chunkwise form of the Gated DeltaNet review,
// meaningful96.github.io/nr/GDN, section 3.7, as read in fwd_simt.cuh).  Per
// chunk, with entry state S (recomputed by the forward and stored per chunk),
// gradient D = dL/dS' of the chunk's exit state, dO of the outputs, and
//     G = strictLower(Gamma * K K^T), A = diag(beta) G, P = (Q K^T) * L,
//     X = K S^T, Y = Q S^T, R = diag(beta)(V - diag(gamma) X), U = (I + A)^-1 R,
//     Kt = diag(exp(g_C - g)) K:
//   dU   = Kt D^T + P^T dO                 dP  = dO U^T (i <= r)
//   dR   = (I + A)^-T dU                   dA  = -dR U^T (i < r)
//   dV   = diag(beta) dR
//   dQ   = diag(gamma) dO S + (dP * L) K
//   dK   = (dP * L)^T Q + dKK K + dKK^T K + diag(exp(g_C - g)) U D - diag(beta gamma) dR S,
//          dKK = dA * beta_r Gamma
//   dbeta_r = sum_c dR_rc (V_rc - gamma_r X_rc) + sum_i dA_ri G_ri
//   dg_r    = gamma_r dO_r.Y_r - beta_r gamma_r dR_r.X_r - exp(g_C-g_r) (U D)_r.K_r
//             + rowsum_r(dP*P) - colsum_r(dP*P) + rowsum_r(dA*A) - colsum_r(dA*A)
//   dg_C   += gamma_C <D, S> + sum_r exp(g_C-g_r) (U D)_r.K_r
//   dS   = gamma_C D + dO^T diag(gamma) Q - dR^T diag(beta gamma) K   (-> D of the previous chunk)
// and finally dlog alpha_s = sum_{r >= s in the chunk} dg_r (g is a prefix sum).
//
// One CTA owns one (b, h) and a slice of kBwdDvs state rows and walks the
// chunks from last to first.  dV and dS are slice-local; dQ, dK, dbeta, dg
// are sums over slices, written per slice to the workspace and summed in a
// fixed order by gdr_bwd_reduce_kernel (deterministic, no atomics).
#pragma once
#include "common.cuh"

#include "fwd_simt.cuh"

namespace gdr {

constexpr int kBwdDvs = 32;  // state rows per CTA

template <int DK>
struct BwdLayout {
    static constexpr int C = kChunk;
    static constexpr int LDK = DK + 1;
    static constexpr int LDV = kBwdDvs + 1;
    static constexpr int LDC = C + 1;
    static constexpr int oQ = 0;
    static constexpr int oK = oQ + C * LDK;
    static constexpr int oS = oK + C * LDK;          // entry state slice  [kBwdDvs][LDK]
    static constexpr int oD = oS + kBwdDvs * LDK;    // dL/dS' slice       [kBwdDvs][LDK]
    static constexpr int oV = oD + kBwdDvs * LDK;    // [C][LDV] each below
    static constexpr int odO = oV + C * LDV;
    static constexpr int oU = odO + C * LDV;
    static constexpr int oX = oU + C * LDV;
    static constexpr int odR = oX + C * LDV;
    static constexpr int oG = odR + C * LDV;         // [C][LDC] each below
    static constexpr int oP = oG + C * LDC;          // P, then dP*P, then dA*A
    static constexpr int odPL = oP + C * LDC;
    static constexpr int odA = odPL + C * LDC;       // dKK
    static constexpr int oGate = odA + C * LDC;      // g, beta, gamma, dec, colsum
    static constexpr int kFloats = oGate + 5 * C + 32;
    static constexpr size_t kBytes = (size_t)kFloats * sizeof(float);
};

// sum over the 16 lanes that share ty (tid = 16 ty + tx, so they are one
// half-warp): deterministic butterfly.
__device__ __forceinline__ float sum16(float x) {
#pragma unroll
    for (int off = 8; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
    return x;
}

// U <- (I + A)^{-1} U, A = diag(beta) G strictly lower; U is C x NC.
template <int LDC, int LDV, int NC>
__device__ __forceinline__ void fwd_solve(const float *sG, const float *sBeta, float *sU) {
    constexpr int kGroups = kSimtThreads / NC;
    constexpr int kRpt = 16 / kGroups;
    const int tid = threadIdx.x;
#pragma unroll 1
    for (int blk = 0; blk < kChunk / 16; ++blk) {
        const int base = blk * 16;
        if (blk > 0) {
            const int c = tid % NC, r0 = base + (tid / NC) * kRpt;
            float acc[kRpt];
#pragma unroll
            for (int a = 0; a < kRpt; ++a) acc[a] = 0.f;
            for (int i = 0; i < base; ++i) {
                const float ui = sU[i * LDV + c];
#pragma unroll
                for (int a = 0; a < kRpt; ++a) acc[a] = fmaf(sG[(r0 + a) * LDC + i], ui, acc[a]);
            }
#pragma unroll
            for (int a = 0; a < kRpt; ++a) sU[(r0 + a) * LDV + c] -= sBeta[r0 + a] * acc[a];
            __syncthreads();
        }
        if (tid < NC) {
            float u[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) u[r] = sU[(base + r) * LDV + tid];
#pragma unroll
            for (int r = 1; r < 16; ++r) {
                float acc = 0.f;
#pragma unroll
                for (int i = 0; i < r; ++i) acc = fmaf(sG[(base + r) * LDC + base + i], u[i], acc);
                u[r] -= sBeta[base + r] * acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sU[(base + r) * LDV + tid] = u[r];
        }
        __syncthreads();
    }
}

// X <- (I + A)^{-T} X, A = diag(beta) G strictly lower: X_r -= sum_{i>r} A_ir X_i.
template <int LDC, int LDV, int NC>
__device__ __forceinline__ void back_solve(const float *sG, const float *sBeta, float *sX) {
    constexpr int kGroups = kSimtThreads / NC;
    constexpr int kRpt = 16 / kGroups;
    const int tid = threadIdx.x;
#pragma unroll 1
    for (int blk = kChunk / 16 - 1; blk >= 0; --blk) {
        const int base = blk * 16;
        if (blk < kChunk / 16 - 1) {
            const int c = tid % NC, r0 = base + (tid / NC) * kRpt;
            float acc[kRpt];
#pragma unroll
            for (int a = 0; a < kRpt; ++a) acc[a] = 0.f;
            for (int i = base + 16; i < kChunk; ++i) {
                const float xi = sBeta[i] * sX[i * LDV + c];
#pragma unroll
                for (int a = 0; a < kRpt; ++a) acc[a] = fmaf(sG[i * LDC + r0 + a], xi, acc[a]);
            }
#pragma unroll
            for (int a = 0; a < kRpt; ++a) sX[(r0 + a) * LDV + c] -= acc[a];
            __syncthreads();
        }
        if (tid < NC) {
            float x[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) x[r] = sX[(base + r) * LDV + tid];
#pragma unroll
            for (int r = 14; r >= 0; --r) {
                float acc = 0.f;
#pragma unroll
                for (int i = r + 1; i < 16; ++i)
                    acc = fmaf(sBeta[base + i] * sG[(base + i) * LDC + base + r], x[i], acc);
                x[r] -= acc;
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sX[(base + r) * LDV + tid] = x[r];
        }
        __syncthreads();
    }
}

template <typename Tio, int DK>
__global__ void __launch_bounds__(kSimtThreads, 1)
gdr_bwd_simt_kernel(int T, int H, int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                    const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                    const float *__restrict__ beta, const Tio *__restrict__ dO,
                    const float *__restrict__ dS_T, const float *__restrict__ S_chunks,
                    Tio *__restrict__ dv_out, float *__restrict__ dS0,
                    float *__restrict__ part_dq, float *__restrict__ part_dk,
                    float *__restrict__ part_db, float *__restrict__ part_dg) {
    using L = BwdLayout<DK>;
    constexpr int NB = DK / 16;
    extern __shared__ float smem[];
    float *sQ = smem + L::oQ, *sK = smem + L::oK, *sS = smem + L::oS, *sD = smem + L::oD;
    float *sV = smem + L::oV, *sdO = smem + L::odO, *sU = smem + L::oU, *sX = smem + L::oX;
    float *sdR = smem + L::odR, *sG = smem + L::oG, *sP = smem + L::oP, *sdPL = smem + L::odPL;
    float *sdA = smem + L::odA;
    float *sg = smem + L::oGate, *sBeta = sg + kChunk, *sGam = sBeta + kChunk;
    float *sDec = sGam + kChunk, *sCol = sDec + kChunk, *sRed = sCol + kChunk;

    const int nslice = dv / kBwdDvs;
    const int slice = blockIdx.x % nslice;
    const int bh = blockIdx.x / nslice;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int vcol0 = slice * kBwdDvs;
    const int nchunks = (T + kChunk - 1) / kChunk;
    const size_t BTH = (size_t)gridDim.x / nslice * T;  // B*H*T token-heads
    const size_t pslice = (size_t)slice * BTH;

    for (int idx = tid; idx < kBwdDvs * DK; idx += blockDim.x) {
        const int r = idx / DK, c = idx % DK;
        sD[r * L::LDK + c] = dS_T ? dS_T[((size_t)bh * dv + vcol0 + r) * DK + c] : 0.f;
    }

#pragma unroll 1
    for (int ch = nchunks - 1; ch >= 0; --ch) {
        const int c0 = ch * kChunk;
        const int n = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        __syncthreads();
        load_tile(sQ, L::LDK, q + tok0 * DK, (size_t)H * DK, n, DK);
        load_tile(sK, L::LDK, k + tok0 * DK, (size_t)H * DK, n, DK);
        load_tile(sV, L::LDV, v + tok0 * dv + vcol0, (size_t)H * dv, n, kBwdDvs);
        load_tile(sdO, L::LDV, dO + tok0 * dv + vcol0, (size_t)H * dv, n, kBwdDvs);
        {
            const float *src = S_chunks + (((size_t)bh * nchunks + ch) * dv + vcol0) * DK;
            for (int idx = tid; idx < kBwdDvs * DK; idx += blockDim.x)
                sS[(idx / DK) * L::LDK + idx % DK] = src[idx];
        }
        chunk_gates(sg, sBeta, sDec, sGam, log_alpha + tok0, beta + tok0, (size_t)H, n);
        __syncthreads();
        const float gamC = sGam[kChunk - 1];

        // per-row gradient accumulators for rows ty + 16a (identical in all 16 lanes of a row)
        float dg_row[4] = {0.f, 0.f, 0.f, 0.f}, db_row[4] = {0.f, 0.f, 0.f, 0.f};

        // ---- P1: G, P (C x C); X = K S^T, Y = Q S^T (C x DVS); R -> sU ----
        {
            float kk[4][4] = {}, qk[4][4] = {}, xs[4][2] = {}, ys[4][2] = {};
#pragma unroll 2
            for (int j = 0; j < DK; ++j) {
                float kr[4], qr[4], ki[4], sc[2];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    kr[a] = sK[(ty + 16 * a) * L::LDK + j];
                    qr[a] = sQ[(ty + 16 * a) * L::LDK + j];
                    ki[a] = sK[(tx + 16 * a) * L::LDK + j];
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) sc[c] = sS[(tx + 16 * c) * L::LDK + j];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        kk[a][c] = fmaf(kr[a], ki[c], kk[a][c]);
                        qk[a][c] = fmaf(qr[a], ki[c], qk[a][c]);
                    }
#pragma unroll
                    for (int c = 0; c < 2; ++c) {
                        xs[a][c] = fmaf(kr[a], sc[c], xs[a][c]);
                        ys[a][c] = fmaf(qr[a], sc[c], ys[a][c]);
                    }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                const float gr = sg[r], br = sBeta[r], gam = sGam[r];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = tx + 16 * c;
                    const float dec = (i <= r) ? expf(gr - sg[i]) : 0.f;
                    sG[r * L::LDC + i] = (i < r) ? dec * kk[a][c] : 0.f;
                    sP[r * L::LDC + i] = dec * qk[a][c];
                }
                float yterm = 0.f;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int cc = tx + 16 * c;
                    sX[r * L::LDV + cc] = xs[a][c];
                    sU[r * L::LDV + cc] = br * (sV[r * L::LDV + cc] - gam * xs[a][c]);
                    yterm = fmaf(sdO[r * L::LDV + cc], ys[a][c], yterm);
                }
                dg_row[a] += gam * sum16(yterm);
            }
        }
        __syncthreads();

        // ---- P2: U = (I + A)^{-1} R ----
        fwd_solve<L::LDC, L::LDV, kBwdDvs>(sG, sBeta, sU);

        // ---- P3a: dU = Kt D^T + P^T dO -> sdR ; dP = dO U^T (registers) ----
        float dp[4][4] = {};
        {
            float du[4][2] = {};
#pragma unroll 2
            for (int j = 0; j < DK; ++j) {
                float kr[4], dd[2];
#pragma unroll
                for (int a = 0; a < 4; ++a) kr[a] = sK[(ty + 16 * a) * L::LDK + j];
#pragma unroll
                for (int c = 0; c < 2; ++c) dd[c] = sD[(tx + 16 * c) * L::LDK + j];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 2; ++c) du[a][c] = fmaf(kr[a], dd[c], du[a][c]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 2; ++c) du[a][c] *= sDec[ty + 16 * a];
#pragma unroll 4
            for (int i = 0; i < kChunk; ++i) {
                float pr[4], od[2];
#pragma unroll
                for (int a = 0; a < 4; ++a) pr[a] = sP[i * L::LDC + ty + 16 * a];
#pragma unroll
                for (int c = 0; c < 2; ++c) od[c] = sdO[i * L::LDV + tx + 16 * c];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 2; ++c) du[a][c] = fmaf(pr[a], od[c], du[a][c]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 2; ++c) sdR[(ty + 16 * a) * L::LDV + tx + 16 * c] = du[a][c];
#pragma unroll 4
            for (int c = 0; c < kBwdDvs; ++c) {
                float od[4], ui[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    od[a] = sdO[(ty + 16 * a) * L::LDV + c];
                    ui[a] = sU[(tx + 16 * a) * L::LDV + c];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) dp[a][cc] = fmaf(od[a], ui[cc], dp[a][cc]);
            }
        }
        __syncthreads();

        // ---- P3b: E = dP * P (row sums now, column sums later), dPL = dP * L ----
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int r = ty + 16 * a;
            float erow = 0.f;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
                const int i = tx + 16 * c;
                const float e = (i <= r) ? dp[a][c] * sP[r * L::LDC + i] : 0.f;
                const float dpl = (i <= r) ? dp[a][c] * expf(sg[r] - sg[i]) : 0.f;
                sP[r * L::LDC + i] = e;
                sdPL[r * L::LDC + i] = dpl;
                erow += e;
            }
            dg_row[a] += sum16(erow);
        }
        __syncthreads();
        if (tid < kChunk) {  // column sums of E
            float s = 0.f;
            for (int r = 0; r < kChunk; ++r) s += sP[r * L::LDC + tid];
            sCol[tid] = s;
        }
        // ---- P4: dR = (I + A)^{-T} dU (in sdR) ----
        back_solve<L::LDC, L::LDV, kBwdDvs>(sG, sBeta, sdR);

        // ---- P5: dA = -dR U^T (strict lower); dbeta / dg row terms; dV ----
        {
            float da[4][4] = {};
#pragma unroll 4
            for (int c = 0; c < kBwdDvs; ++c) {
                float dr[4], ui[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    dr[a] = sdR[(ty + 16 * a) * L::LDV + c];
                    ui[a] = sU[(tx + 16 * a) * L::LDV + c];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int cc = 0; cc < 4; ++cc) da[a][cc] = fmaf(-dr[a], ui[cc], da[a][cc]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                const float br = sBeta[r];
                float frow = 0.f;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = tx + 16 * c;
                    float f = 0.f, dkk = 0.f, fb = 0.f;
                    if (i < r) {
                        f = da[a][c] * sG[r * L::LDC + i];
                        fb = br * f;
                        dkk = da[a][c] * br * expf(sg[r] - sg[i]);
                    }
                    sP[r * L::LDC + i] = fb;   // dA * A, for the column sums
                    sdA[r * L::LDC + i] = dkk;
                    frow += f;
                }
                frow = sum16(frow);
                db_row[a] += frow;
                dg_row[a] += br * frow;
                // X / V terms of dbeta and dg (slice-local columns)
                float bx = 0.f, gx = 0.f;
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int cc = tx + 16 * c;
                    const float dr = sdR[r * L::LDV + cc], xv = sX[r * L::LDV + cc];
                    bx = fmaf(dr, sV[r * L::LDV + cc] - sGam[r] * xv, bx);
                    gx = fmaf(dr, xv, gx);
                    if (r < n)
                        dv_out[(tok0 + (size_t)r * H) * dv + vcol0 + cc] = from_f32<Tio>(br * dr);
                }
                db_row[a] += sum16(bx);
                dg_row[a] -= br * sGam[r] * sum16(gx);
            }
        }
        __syncthreads();
        if (tid < kChunk) {  // column sums of dA * A
            float s = 0.f;
            for (int r = 0; r < kChunk; ++r) s += sP[r * L::LDC + tid];
            sCol[tid] += s;
        }

        // ---- P6: dK, dQ (C x DK) and the new D ----
        float zpart = 0.f;  // exp(g_C-g_r)(U D)_r.K_r summed over this thread's rows (for dg_C)
        {
            float acc[4][NB] = {};
            // U D (C x DK) -> diag(dec) U D, and its z terms
#pragma unroll 4
            for (int c = 0; c < kBwdDvs; ++c) {
                float ur[4], dd[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) ur[a] = sU[(ty + 16 * a) * L::LDV + c];
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) dd[bq] = sD[c * L::LDK + tx + 16 * bq];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) acc[a][bq] = fmaf(ur[a], dd[bq], acc[a][bq]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                const float dec = sDec[r];
                float z = 0.f;
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    acc[a][bq] *= dec;
                    z = fmaf(acc[a][bq], sK[r * L::LDK + tx + 16 * bq], z);
                }
                z = sum16(z);
                dg_row[a] -= z;
                if (tx == 0) zpart += z;
            }
            // - diag(beta gamma) dR S
#pragma unroll 4
            for (int c = 0; c < kBwdDvs; ++c) {
                float dr[4], ss[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = ty + 16 * a;
                    dr[a] = -sBeta[r] * sGam[r] * sdR[r * L::LDV + c];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) ss[bq] = sS[c * L::LDK + tx + 16 * bq];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) acc[a][bq] = fmaf(dr[a], ss[bq], acc[a][bq]);
            }
            // (dP*L)^T Q + dKK K + dKK^T K
#pragma unroll 2
            for (int i = 0; i < kChunk; ++i) {
                float w1[4], w2[4], w3[4], qi[NB], ki[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = ty + 16 * a;
                    w1[a] = sdPL[i * L::LDC + r];
                    w2[a] = sdA[r * L::LDC + i];
                    w3[a] = sdA[i * L::LDC + r];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    qi[bq] = sQ[i * L::LDK + tx + 16 * bq];
                    ki[bq] = sK[i * L::LDK + tx + 16 * bq];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq)
                        acc[a][bq] = fmaf(w1[a], qi[bq], fmaf(w2[a] + w3[a], ki[bq], acc[a][bq]));
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                float *dst = part_dk + pslice * DK + (tok0 + (size_t)r * H) * DK;
                if (r < n)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) dst[tx + 16 * bq] = acc[a][bq];
            }
        }
        {
            float acc[4][NB] = {};
            // diag(gamma) dO S + (dP*L) K
#pragma unroll 4
            for (int c = 0; c < kBwdDvs; ++c) {
                float od[4], ss[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = ty + 16 * a;
                    od[a] = sGam[r] * sdO[r * L::LDV + c];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) ss[bq] = sS[c * L::LDK + tx + 16 * bq];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) acc[a][bq] = fmaf(od[a], ss[bq], acc[a][bq]);
            }
#pragma unroll 4
            for (int i = 0; i < kChunk; ++i) {
                float w[4], ki[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) w[a] = sdPL[(ty + 16 * a) * L::LDC + i];
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) ki[bq] = sK[i * L::LDK + tx + 16 * bq];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) acc[a][bq] = fmaf(w[a], ki[bq], acc[a][bq]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                float *dst = part_dq + pslice * DK + (tok0 + (size_t)r * H) * DK;
                if (r < n)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) dst[tx + 16 * bq] = acc[a][bq];
            }
        }
        // new D = gamma_C D + dO^T diag(gamma) Q - dR^T diag(beta gamma) K, and gamma_C <D, S>
        float dS_new[2][NB];
        float dsum = 0.f;
        {
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    const int c = ty + 16 * a, j = tx + 16 * bq;
                    const float dcur = sD[c * L::LDK + j];
                    dsum = fmaf(dcur, sS[c * L::LDK + j], dsum);
                    dS_new[a][bq] = gamC * dcur;
                }
#pragma unroll 4
            for (int r = 0; r < kChunk; ++r) {
                const float gr = sGam[r], bgr = sBeta[r] * gr;
                float w1[2], w2[2], qr[NB], kr[NB];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    w1[a] = gr * sdO[r * L::LDV + ty + 16 * a];
                    w2[a] = -bgr * sdR[r * L::LDV + ty + 16 * a];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    qr[bq] = sQ[r * L::LDK + tx + 16 * bq];
                    kr[bq] = sK[r * L::LDK + tx + 16 * bq];
                }
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq)
                        dS_new[a][bq] = fmaf(w1[a], qr[bq], fmaf(w2[a], kr[bq], dS_new[a][bq]));
            }
        }
        // block reduction of gamma_C <D,S> + sum z (fixed order: deterministic)
        {
            float x = gamC * dsum + zpart;
#pragma unroll
            for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
            if ((tid & 31) == 0) sRed[tid >> 5] = x;
        }
        __syncthreads();  // every read of D, S, sCol writers done
#pragma unroll
        for (int a = 0; a < 2; ++a)
#pragma unroll
            for (int bq = 0; bq < NB; ++bq) sD[(ty + 16 * a) * L::LDK + tx + 16 * bq] = dS_new[a][bq];
        if (tx == 0) {
            float dgC = 0.f;
            for (int w = 0; w < kSimtThreads / 32; ++w) dgC += sRed[w];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                if (r < n) {
                    float dg = dg_row[a] - sCol[r];
                    if (r == n - 1) dg += dgC;
                    part_dg[pslice + tok0 + (size_t)r * H] = dg;
                    part_db[pslice + tok0 + (size_t)r * H] = db_row[a];
                }
            }
        }
    }
    __syncthreads();
    if (dS0) {
        for (int idx = tid; idx < kBwdDvs * DK; idx += blockDim.x) {
            const int r = idx / DK, c = idx % DK;
            dS0[((size_t)bh * dv + vcol0 + r) * DK + c] = sD[r * L::LDK + c];
        }
    }
}

// Sum the per-slice partials in a fixed order; dlog alpha = reverse prefix
// sum of dg inside each chunk.  One CTA per (b, h, chunk).
template <typename Tio, int DK>
__global__ void __launch_bounds__(256)
gdr_bwd_reduce_kernel(int T, int H, int nslice, const float *__restrict__ part_dq,
                      const float *__restrict__ part_dk, const float *__restrict__ part_db,
                      const float *__restrict__ part_dg, Tio *__restrict__ dq, Tio *__restrict__ dk,
                      float *__restrict__ dlog_alpha, float *__restrict__ dbeta, size_t BTH) {
    const int nchunks = (T + kChunk - 1) / kChunk;
    const int ch = blockIdx.x % nchunks;
    const int bh = blockIdx.x / nchunks;
    const int b = bh / H, h = bh % H;
    const int c0 = ch * kChunk, n = min(kChunk, T - c0);
    const size_t tok0 = ((size_t)b * T + c0) * H + h;
    for (int idx = threadIdx.x; idx < n * DK; idx += blockDim.x) {
        const int r = idx / DK, j = idx % DK;
        const size_t off = (tok0 + (size_t)r * H) * DK + j;
        float sq = 0.f, sk = 0.f;
        for (int s = 0; s < nslice; ++s) {
            sq += part_dq[(size_t)s * BTH * DK + off];
            sk += part_dk[(size_t)s * BTH * DK + off];
        }
        dq[off] = from_f32<Tio>(sq);
        dk[off] = from_f32<Tio>(sk);
    }
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        float g[2], bsum[2];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
            const int r = 2 * lane + e;
            g[e] = 0.f;
            bsum[e] = 0.f;
            if (r < n) {
                const size_t off = tok0 + (size_t)r * H;
                for (int s = 0; s < nslice; ++s) {
                    g[e] += part_dg[(size_t)s * BTH + off];
                    bsum[e] += part_db[(size_t)s * BTH + off];
                }
            }
        }
        // reverse inclusive prefix sum over r = 0..63 (lane holds rows 2l, 2l+1)
        float pair = g[0] + g[1];
        float suffix = pair;  // sum over lanes >= lane
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_down_sync(0xffffffffu, suffix, off);
            if (lane + off < 32) suffix += y;
        }
        const float after = suffix - pair;  // rows > 2l+1
        const float d1 = after + g[1], d0 = d1 + g[0];
        if (2 * lane < n) {
            dlog_alpha[tok0 + (size_t)(2 * lane) * H] = d0;
            dbeta[tok0 + (size_t)(2 * lane) * H] = bsum[0];
        }
        if (2 * lane + 1 < n) {
            dlog_alpha[tok0 + (size_t)(2 * lane + 1) * H] = d1;
            dbeta[tok0 + (size_t)(2 * lane + 1) * H] = bsum[1];
        }
    }
}

struct BwdWorkspace {
    float *states, *part_dq, *part_dk, *part_db, *part_dg;
};

inline size_t bwd_workspace_bytes(int B, int T, int H, int dk, int dv) {
    const size_t nch = (size_t)(T + kChunk - 1) / kChunk;
    const size_t ns = (size_t)dv / kBwdDvs;
    const size_t bth = (size_t)B * T * H;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    return al((size_t)B * H * nch * dv * dk * 4) + 2 * al(ns * bth * dk * 4) + 2 * al(ns * bth * 4);
}

inline BwdWorkspace bwd_carve(void *ws, int B, int T, int H, int dk, int dv) {
    const size_t nch = (size_t)(T + kChunk - 1) / kChunk;
    const size_t ns = (size_t)dv / kBwdDvs;
    const size_t bth = (size_t)B * T * H;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    char *p = static_cast<char *>(ws);
    BwdWorkspace w;
    w.states = reinterpret_cast<float *>(p);
    p += al((size_t)B * H * nch * dv * dk * 4);
    w.part_dq = reinterpret_cast<float *>(p);
    p += al(ns * bth * dk * 4);
    w.part_dk = reinterpret_cast<float *>(p);
    p += al(ns * bth * dk * 4);
    w.part_db = reinterpret_cast<float *>(p);
    p += al(ns * bth * 4);
    w.part_dg = reinterpret_cast<float *>(p);
    return w;
}

template <typename Tio, int DK>
cudaError_t launch_bwd_simt(int B, int T, int H, int dv, const void *q, const void *k,
                            const void *v, const float *la, const float *beta, const float *S0,
                            const void *dO, const float *dS_T, void *dq, void *dk_out,
                            void *dv_out, float *dla, float *dbeta, float *dS0, void *ws,
                            cudaStream_t stream) {
    BwdWorkspace w = bwd_carve(ws, B, T, H, DK, dv);
    // 1) forward recompute on the CUDA cores, keeping every chunk's fp32 entry
    //    state (this backward is also the cross-check of the tensor-core one,
    //    so it shares none of its kernels)
    cudaError_t err = launch_fwd_simt<Tio, DK>(B, T, H, dv, q, k, v, la, beta, S0, nullptr, nullptr, stream,
                                               w.states);
    if (err != cudaSuccess) return err;
    // 2) reverse chunk pass per (b, h, slice)
    using L = BwdLayout<DK>;
    auto kern = gdr_bwd_simt_kernel<Tio, DK>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (err != cudaSuccess) return err;
    const int nslice = dv / kBwdDvs;
    kern<<<(unsigned)(B * H * nslice), kSimtThreads, L::kBytes, stream>>>(
        T, H, dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k),
        static_cast<const Tio *>(v), la, beta, static_cast<const Tio *>(dO), dS_T, w.states,
        static_cast<Tio *>(dv_out), dS0, w.part_dq, w.part_dk, w.part_db, w.part_dg);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    // 3) sum the slices, dlog alpha by reverse prefix sums
    const int nch = (T + kChunk - 1) / kChunk;
    gdr_bwd_reduce_kernel<Tio, DK><<<(unsigned)(B * H * nch), 256, 0, stream>>>(
        T, H, nslice, w.part_dq, w.part_dk, w.part_db, w.part_dg, static_cast<Tio *>(dq),
        static_cast<Tio *>(dk_out), dla, dbeta, (size_t)B * T * H);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
