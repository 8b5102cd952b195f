// gdr2_simt.cuh -- chunkwise Gated DeltaNet-2 forward on CUDA cores (fp32).
//
// Gated Delta Rule-2 ("Gated DeltaNet-2: Decoupling Erase and Write in Linear
// Attention", agihunt.info/papers/2605.22791): per token, decay each key
// channel by alpha_t, read the old value along b_t*k_t, write the residual of
// w_t*v_t along k_t:  S' = S Diag(alpha_t);  S_t = S' - (S'(b_t*k_t) - w_t*v_t) k_t^T.
// The page's chunkwise statement: the channel decay is absorbed into an
// asymmetric rank-1 erase factor and each 64-token chunk is still a WY
// triangular solve plus dense products.  With per-channel cumulative log
// decay G_r = sum_{s<=r} log alpha_s (a C x dk matrix):
//     A_ri = sum_j b_r[j] k_r[j] k_i[j] exp(G_r[j] - G_i[j])      (i < r)
//     U    = (I + A)^{-1} (W*V - (K*B*exp(G)) S^T)
//     O    = (Q*exp(G)) S^T + P U,  P_ri = sum_j q_r[j] k_i[j] exp(G_r[j] - G_i[j])  (i <= r)
//     S'   = S Diag(exp(G_C)) + U^T (K * exp(G_C - G))
// The decay ratios exp(G_r[j] - G_i[j]) enter the products through operands
// scaled about the chunk's middle token: Q*E', K*B*E' and K/E' with
// E' = exp(G - G_31) per (token, channel), so the dot products carry no
// exponential; S is scaled by exp(G_31) on the fly for the S products and the
// state update uses K/E' times exp(G_C - G_31).  A chunk in which some
// channel decays by more than e^80 (where E' or 1/E' could overflow) takes
// the exact path, which evaluates exp(G_r[j] - G_i[j]) per element.  Same
// CTA / slice structure as fwd_simt.cuh.
#pragma once
#include "common.cuh"
#include "fwd_simt.cuh"

namespace gdr {

template <int DK>
struct Gdr2Layout {
    static constexpr int C = kChunk;
    static constexpr int LDK = DK + 1;
    static constexpr int LDV = kSimtDvs + 1;
    static constexpr int LDC = C + 1;
    static constexpr int oQ = 0;
    static constexpr int oK = oQ + C * LDK;
    static constexpr int oKB = oK + C * LDK;   // K * b
    static constexpr int oG = oKB + C * LDK;   // cumulative log decay per channel
    static constexpr int oS = oG + C * LDK;
    static constexpr int oU = oS + kSimtDvs * LDK;
    static constexpr int oA = oU + C * LDV;
    static constexpr int oP = oA + C * LDC;
    static constexpr int oVec = oP + C * LDC;  // exp(G_31), exp(G_C), exp(G_C - G_31) per channel; flag
    static constexpr int kFloats = oVec + 3 * DK + 4;
    static constexpr size_t kBytes = (size_t)kFloats * sizeof(float);
};

template <typename Tio, int DK>
__global__ void __launch_bounds__(kSimtThreads, 1)
gdr2_fwd_simt_kernel(int T, int H, int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                     const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ bgate, const float *__restrict__ wgate,
                     const float *__restrict__ S0, Tio *__restrict__ o, float *__restrict__ S_T,
                     float *__restrict__ S_chunks) {
    using L = Gdr2Layout<DK>;
    constexpr int NB = DK / 16;
    extern __shared__ float smem[];
    float *sQ = smem + L::oQ, *sK = smem + L::oK, *sKB = smem + L::oKB, *sG = smem + L::oG;
    float *sS = smem + L::oS, *sU = smem + L::oU, *sA = smem + L::oA, *sP = smem + L::oP;
    float *sE31 = smem + L::oVec, *sEC = sE31 + DK, *sEpC = sEC + DK;
    int *s_exact = reinterpret_cast<int *>(sEpC + DK);

    const int nslice = dv / kSimtDvs;
    const int slice = blockIdx.x % nslice;
    const int bh = blockIdx.x / nslice;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int vcol0 = slice * kSimtDvs;

    for (int idx = tid; idx < kSimtDvs * DK; idx += blockDim.x) {
        const int r = idx / DK, c = idx % DK;
        sS[r * L::LDK + c] = S0 ? S0[((size_t)bh * dv + vcol0 + r) * DK + c] : 0.f;
    }

#pragma unroll 1
    for (int c0 = 0; c0 < T; c0 += kChunk) {
        const int n = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        __syncthreads();
        load_tile(sQ, L::LDK, q + tok0 * DK, (size_t)H * DK, n, DK);
        load_tile(sK, L::LDK, k + tok0 * DK, (size_t)H * DK, n, DK);
        if (S_chunks) {  // chunk-entry state for the backward's recompute pass
            float *dst = S_chunks + (((size_t)bh * ((T + kChunk - 1) / kChunk) + c0 / kChunk) * dv + vcol0) * DK;
            for (int idx = tid; idx < kSimtDvs * DK; idx += blockDim.x)
                dst[idx] = sS[(idx / DK) * L::LDK + idx % DK];
        }
        // R <- w * v (slice columns), zero past the end
        for (int idx = tid; idx < kChunk * kSimtDvs; idx += blockDim.x) {
            const int r = idx / kSimtDvs, c = idx % kSimtDvs;
            float x = 0.f;
            if (r < n) {
                const size_t off = (tok0 + (size_t)r * H) * dv + vcol0 + c;
                x = wgate[off] * to_f32(v[off]);
            }
            sU[r * L::LDV + c] = x;
        }
        __syncthreads();
        // per-channel cumulative log decay (padded rows: log alpha = 0) and K * b
        for (int j = tid; j < DK; j += blockDim.x) {
            float g = 0.f;
            for (int r = 0; r < kChunk; ++r) {
                float la = 0.f, bg = 0.f;
                if (r < n) {
                    const size_t off = (tok0 + (size_t)r * H) * DK + j;
                    la = log_alpha[off];
                    bg = bgate[off];
                }
                g += la;
                sG[r * L::LDK + j] = g;
                sKB[r * L::LDK + j] = bg * sK[r * L::LDK + j];
            }
        }
        if (tid == 0) *s_exact = 0;
        __syncthreads();
        for (int j = tid; j < DK; j += blockDim.x) {
            const float g0 = sG[j], gM = sG[31 * L::LDK + j], gC = sG[(kChunk - 1) * L::LDK + j];
            if (g0 - gC > 80.f) *s_exact = 1;
            sE31[j] = expf(gM);
            sEC[j] = expf(gC);
            sEpC[j] = expf(gC - gM);
        }
        __syncthreads();
        const bool exact = *s_exact != 0;
        if (!exact) {  // Q*E', (K*B)*E', K/E' with E' = exp(G - G_31)
            for (int idx = tid; idx < kChunk * DK; idx += blockDim.x) {
                const int r = idx / DK, j = idx % DK;
                const float d = sG[r * L::LDK + j] - sG[31 * L::LDK + j];
                const float e = __expf(d), ie = __expf(-d);
                sQ[r * L::LDK + j] *= e;
                sKB[r * L::LDK + j] *= e;
                sK[r * L::LDK + j] *= ie;
            }
            __syncthreads();
        }

        // ---- phase 1: A, P (decay inside the dot products); X, Y against S ----
        float o_acc[4][4];
        {
            float aa[4][4] = {}, pp[4][4] = {}, xs[4][4] = {};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) o_acc[a][c] = 0.f;
            if (exact) {
#pragma unroll 2
            for (int j = 0; j < DK; ++j) {
                float kbr[4], qr[4], gr[4], ki[4], gi[4], sc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    kbr[a] = sKB[(ty + 16 * a) * L::LDK + j];
                    qr[a] = sQ[(ty + 16 * a) * L::LDK + j];
                    gr[a] = sG[(ty + 16 * a) * L::LDK + j];
                    ki[a] = sK[(tx + 16 * a) * L::LDK + j];
                    gi[a] = sG[(tx + 16 * a) * L::LDK + j];
                    sc[a] = sS[(tx + 16 * a) * L::LDK + j];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const float er = expf(gr[a]);
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        // ratio exp(G_r - G_i) <= 1 for i <= r; clamp keeps masked pairs finite
                        const float ratio = expf(fminf(gr[a] - gi[c], 0.f)) * ki[c];
                        aa[a][c] = fmaf(kbr[a], ratio, aa[a][c]);
                        pp[a][c] = fmaf(qr[a], ratio, pp[a][c]);
                        xs[a][c] = fmaf(kbr[a] * er, sc[c], xs[a][c]);
                        o_acc[a][c] = fmaf(qr[a] * er, sc[c], o_acc[a][c]);
                    }
                }
            }
            } else {
#pragma unroll 4
                for (int j = 0; j < DK; ++j) {
                    float kbr[4], qr[4], ki[4], sc[4];
                    const float e31 = sE31[j];
#pragma unroll
                    for (int a = 0; a < 4; ++a) {
                        kbr[a] = sKB[(ty + 16 * a) * L::LDK + j];
                        qr[a] = sQ[(ty + 16 * a) * L::LDK + j];
                        ki[a] = sK[(tx + 16 * a) * L::LDK + j];
                        sc[a] = sS[(tx + 16 * a) * L::LDK + j] * e31;
                    }
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            aa[a][c] = fmaf(kbr[a], ki[c], aa[a][c]);
                            pp[a][c] = fmaf(qr[a], ki[c], pp[a][c]);
                            xs[a][c] = fmaf(kbr[a], sc[c], xs[a][c]);
                            o_acc[a][c] = fmaf(qr[a], sc[c], o_acc[a][c]);
                        }
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = tx + 16 * c;
                    sA[r * L::LDC + i] = (i < r) ? aa[a][c] : 0.f;
                    sP[r * L::LDC + i] = (i <= r) ? pp[a][c] : 0.f;
                    sU[r * L::LDV + i] -= xs[a][c];
                }
            }
        }
        __syncthreads();

        // ---- phase 2: U = (I + A)^{-1} R ----
        solve_unit_lower<L::LDC, L::LDV>(sA, sU);

        // ---- phase 3: O += P U ----
#pragma unroll 4
        for (int i = 0; i < kChunk; ++i) {
            float pr[4], ui[4];
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                pr[a] = sP[(ty + 16 * a) * L::LDC + i];
                ui[a] = sU[i * L::LDV + tx + 16 * a];
            }
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) o_acc[a][c] = fmaf(pr[a], ui[c], o_acc[a][c]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int r = ty + 16 * a;
            if (r < n && o) {
                Tio *orow = o + (tok0 + (size_t)r * H) * dv + vcol0;
#pragma unroll
                for (int c = 0; c < 4; ++c) orow[tx + 16 * c] = from_f32<Tio>(o_acc[a][c]);
            }
        }

        // ---- phase 4: S <- S Diag(exp(G_C)) + U^T (K * exp(G_C - G)) ----
        {
            float acc[4][NB];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < NB; ++c) acc[a][c] = 0.f;
            float gC[NB];
#pragma unroll
            for (int c = 0; c < NB; ++c) gC[c] = sG[(kChunk - 1) * L::LDK + tx + 16 * c];
#pragma unroll 2
            for (int r = 0; r < kChunk; ++r) {
                float ur[4], kr[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) ur[a] = sU[r * L::LDV + ty + 16 * a];
#pragma unroll
                for (int c = 0; c < NB; ++c) {
                    const int j = tx + 16 * c;
                    // exact: k * exp(G_C - G_r); scaled: (K/E') times exp(G_C - G_31), applied below
                    kr[c] = exact ? sK[r * L::LDK + j] * expf(gC[c] - sG[r * L::LDK + j]) : sK[r * L::LDK + j];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < NB; ++c) acc[a][c] = fmaf(ur[a], kr[c], acc[a][c]);
            }
            if (!exact) {
#pragma unroll
                for (int c = 0; c < NB; ++c) {
                    const float f = sEpC[tx + 16 * c];
#pragma unroll
                    for (int a = 0; a < 4; ++a) acc[a][c] *= f;
                }
            }
            __syncthreads();  // everyone finished reading S (phase 1) and U
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < NB; ++c) {
                    float *s = &sS[(ty + 16 * a) * L::LDK + tx + 16 * c];
                    *s = fmaf(expf(gC[c]), *s, acc[a][c]);
                }
        }
    }
    __syncthreads();
    if (S_T) {
        for (int idx = tid; idx < kSimtDvs * DK; idx += blockDim.x) {
            const int r = idx / DK, c = idx % DK;
            S_T[((size_t)bh * dv + vcol0 + r) * DK + c] = sS[r * L::LDK + c];
        }
    }
}

template <typename Tio, int DK>
// o == nullptr skips the outputs (the backward's recompute); S_chunks
// (nullable) receives every chunk's entry state, [B, H, nchunks, dv, DK] fp32.
cudaError_t launch_gdr2_simt(int B, int T, int H, int dv, const void *q, const void *k,
                             const void *v, const float *la, const float *bg, const float *wg,
                             const float *S0, void *o, float *S_T, cudaStream_t stream,
                             float *S_chunks = nullptr) {
    using L = Gdr2Layout<DK>;
    auto kern = gdr2_fwd_simt_kernel<Tio, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)L::kBytes);
    if (err != cudaSuccess) return err;
    kern<<<(unsigned)(B * H * (dv / kSimtDvs)), kSimtThreads, L::kBytes, stream>>>(
        T, H, dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k),
        static_cast<const Tio *>(v), la, bg, wg, S0, static_cast<Tio *>(o), S_T, S_chunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
