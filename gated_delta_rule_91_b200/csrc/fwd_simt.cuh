// fwd_simt.cuh -- chunkwise forward on CUDA cores in fp32 (gdr_fwd for fp32
// inputs, and for shapes the tensor-core kernel does not take).
//
// Chunkwise form of the gated delta rule (Gated DeltaNet review,
// meaningful96.github.io/nr/GDN, section 3.7, read with the decay on the
// intra-chunk mask and W = T diag(beta*gamma) K).  Per chunk of C = 64 tokens
// with g_r = sum_{s<=r} log alpha_s, gamma_r = exp(g_r) and entry state S:
//     A  = strictLower(diag(beta)(Gamma * K K^T)),  Gamma_ri = exp(g_r - g_i)
//     U  = (I + A)^{-1} diag(beta)(V - diag(gamma) K S^T)      (= U^g - W S^T)
//     O  = diag(gamma) Q S^T + (Q K^T * L) U,        L_ri = exp(g_r - g_i), i <= r
//     S' = gamma_C S + U^T diag(exp(g_C - g)) K
// U is found by blocked forward substitution in shared memory (16-row
// diagonal blocks solved column-per-thread, off-diagonal updates as small
// matmuls), which is the same lower-triangular solve as forming the UT
// matrix T = (I + A)^{-1} first.
//
// One CTA owns one (b, h) and a slice of kDvs state rows; rows of S evolve
// independently, so slices need no communication.  The slice's state stays
// in shared memory (fp32) for the whole sequence.  Tokens past T in the last
// chunk are padded as identity steps (k = q = v = 0, log alpha = 0, beta = 0).
#pragma once
#include "common.cuh"

namespace gdr {

constexpr int kSimtThreads = 256;
constexpr int kSimtDvs = 64;  // state rows per CTA

template <int DK>
struct FwdSimtLayout {
    static constexpr int C = kChunk;
    static constexpr int LDK = DK + 1;        // row stride of Q, K, S tiles (odd: no bank conflicts)
    static constexpr int LDV = kSimtDvs + 1;  // row stride of V, U tiles
    static constexpr int LDC = C + 1;         // row stride of A, P
    static constexpr int oQ = 0;
    static constexpr int oK = oQ + C * LDK;
    static constexpr int oS = oK + C * LDK;
    static constexpr int oV = oS + kSimtDvs * LDK;
    static constexpr int oU = oV + C * LDV;
    static constexpr int oA = oU + C * LDV;
    static constexpr int oP = oA + C * LDC;
    static constexpr int oG = oP + C * LDC;   // g_r
    static constexpr int oB = oG + C;         // beta_r
    static constexpr int oDec = oB + C;       // exp(g_C - g_r)
    static constexpr int oGam = oDec + C;     // gamma_r
    static constexpr int kFloats = oGam + C;
    static constexpr size_t kBytes = (size_t)kFloats * sizeof(float);
};

// Load rows [c0, c0+C) of a [*, rowstride] token-major tensor (columns
// [col0, col0+ncols)) into fp32 shared memory with row stride ld; rows at or
// past n are zero.
template <typename Tio>
__device__ __forceinline__ void load_tile(float *dst, int ld, const Tio *src, size_t rowstride,
                                          int n, int ncols) {
    const int vecs_per_row = ncols / 8;
    for (int idx = threadIdx.x; idx < kChunk * vecs_per_row; idx += blockDim.x) {
        const int r = idx / vecs_per_row, c = (idx % vecs_per_row) * 8;
        float tmp[8];
        if (r < n) {
            load8(src + (size_t)r * rowstride + c, tmp);
        } else {
#pragma unroll
            for (int i = 0; i < 8; ++i) tmp[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[r * ld + c + i] = tmp[i];
    }
}

// Per-chunk gate preparation: g (inclusive cumulative log-decay), gamma,
// exp(g_C - g_r), beta; padded rows get log alpha = 0, beta = 0.
__device__ __forceinline__ void chunk_gates(float *sG, float *sB, float *sDec, float *sGam,
                                            const float *la, const float *beta, size_t stride,
                                            int n) {
    if (threadIdx.x < 32) {
        const int lane = threadIdx.x;
        const int r0 = 2 * lane, r1 = 2 * lane + 1;
        const float l0 = r0 < n ? la[(size_t)r0 * stride] : 0.f;
        const float l1 = r1 < n ? la[(size_t)r1 * stride] : 0.f;
        float incl = l0 + l1;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const float y = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off) incl += y;
        }
        const float g1 = incl, g0 = incl - l1;
        const float gC = __shfl_sync(0xffffffffu, incl, 31);
        sG[r0] = g0;
        sG[r1] = g1;
        sGam[r0] = expf(g0);
        sGam[r1] = expf(g1);
        sDec[r0] = expf(gC - g0);
        sDec[r1] = expf(gC - g1);
        sB[r0] = r0 < n ? beta[(size_t)r0 * stride] : 0.f;
        sB[r1] = r1 < n ? beta[(size_t)r1 * stride] : 0.f;
    }
}

// Blocked forward substitution: U <- (I + A)^{-1} U in place (A strictly
// lower, 64 x 64, row stride LDC; U 64 x kSimtDvs, row stride LDV).
template <int LDC, int LDV>
__device__ __forceinline__ void solve_unit_lower(const float *sA, float *sU) {
    const int tid = threadIdx.x;
#pragma unroll 1
    for (int blk = 0; blk < kChunk / 16; ++blk) {
        const int base = blk * 16;
        if (blk > 0) {
            // rows base..base+15 -= A[rows, 0:base] U[0:base, :]
            const int c = tid % kSimtDvs;
            const int rq = (tid / kSimtDvs) * 4;  // 4 rows per thread
            float acc[4] = {0.f, 0.f, 0.f, 0.f};
            for (int i = 0; i < base; ++i) {
                const float ui = sU[i * LDV + c];
#pragma unroll
                for (int a = 0; a < 4; ++a) acc[a] = fmaf(sA[(base + rq + a) * LDC + i], ui, acc[a]);
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) sU[(base + rq + a) * LDV + c] -= acc[a];
            __syncthreads();
        }
        if (tid < kSimtDvs) {
            float u[16];
#pragma unroll
            for (int r = 0; r < 16; ++r) u[r] = sU[(base + r) * LDV + tid];
#pragma unroll
            for (int r = 1; r < 16; ++r) {
#pragma unroll
                for (int i = 0; i < r; ++i) u[r] = fmaf(-sA[(base + r) * LDC + base + i], u[i], u[r]);
            }
#pragma unroll
            for (int r = 0; r < 16; ++r) sU[(base + r) * LDV + tid] = u[r];
        }
        __syncthreads();
    }
}

template <typename Tio, int DK>
__global__ void __launch_bounds__(kSimtThreads, 1)
gdr_fwd_simt_kernel(int T, int H, int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                    const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                    const float *__restrict__ beta, const float *__restrict__ S0,
                    Tio *__restrict__ o, float *__restrict__ S_T,
                    float *__restrict__ S_chunks) {
    using L = FwdSimtLayout<DK>;
    extern __shared__ float smem[];
    float *sQ = smem + L::oQ, *sK = smem + L::oK, *sS = smem + L::oS, *sV = smem + L::oV;
    float *sU = smem + L::oU, *sA = smem + L::oA, *sP = smem + L::oP;
    float *sG = smem + L::oG, *sB = smem + L::oB, *sDec = smem + L::oDec, *sGam = smem + L::oGam;

    const int nslice = dv / kSimtDvs;
    const int slice = blockIdx.x % nslice;
    const int bh = blockIdx.x / nslice;
    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int vcol0 = slice * kSimtDvs;

    // entry state of this slice
    for (int idx = tid; idx < kSimtDvs * DK; idx += blockDim.x) {
        const int r = idx / DK, c = idx % DK;
        sS[r * L::LDK + c] = S0 ? S0[((size_t)bh * dv + vcol0 + r) * DK + c] : 0.f;
    }

    const size_t tokstride = (size_t)H;  // between consecutive tokens in [B,T,H]
    for (int c0 = 0; c0 < T; c0 += kChunk) {
        const int n = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        __syncthreads();  // previous chunk is done with every tile
        if (S_chunks) {  // chunk-entry state for the backward's recompute pass
            float *dst = S_chunks + (((size_t)bh * ((T + kChunk - 1) / kChunk) + c0 / kChunk) * dv + vcol0) * DK;
            for (int idx = tid; idx < kSimtDvs * DK; idx += blockDim.x)
                dst[idx] = sS[(idx / DK) * L::LDK + idx % DK];
        }
        load_tile(sQ, L::LDK, q + tok0 * DK, (size_t)H * DK, n, DK);
        load_tile(sK, L::LDK, k + tok0 * DK, (size_t)H * DK, n, DK);
        load_tile(sV, L::LDV, v + tok0 * dv + vcol0, (size_t)H * dv, n, kSimtDvs);
        chunk_gates(sG, sB, sDec, sGam, log_alpha + tok0, beta + tok0, tokstride, n);
        __syncthreads();

        // ---- phase 1: KK^T, QK^T (-> A, P), K S^T (-> R), Q S^T (-> O, kept) ----
        float o_acc[4][4];
        {
            float kk[4][4] = {}, qk[4][4] = {}, xs[4][4] = {};
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 4; ++c) o_acc[a][c] = 0.f;
#pragma unroll 4
            for (int j = 0; j < DK; ++j) {
                float kr[4], qr[4], ki[4], sc[4];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    kr[a] = sK[(ty + 16 * a) * L::LDK + j];
                    qr[a] = sQ[(ty + 16 * a) * L::LDK + j];
                    ki[a] = sK[(tx + 16 * a) * L::LDK + j];
                    sc[a] = sS[(tx + 16 * a) * L::LDK + j];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        kk[a][c] = fmaf(kr[a], ki[c], kk[a][c]);
                        qk[a][c] = fmaf(qr[a], ki[c], qk[a][c]);
                        xs[a][c] = fmaf(kr[a], sc[c], xs[a][c]);
                        o_acc[a][c] = fmaf(qr[a], sc[c], o_acc[a][c]);
                    }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                const float gr = sG[r], br = sB[r], gam = sGam[r];
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = tx + 16 * c;  // key index for A/P, value column for R/O
                    const float dec = (i <= r) ? expf(gr - sG[i]) : 0.f;
                    sA[r * L::LDC + i] = (i < r) ? br * dec * kk[a][c] : 0.f;
                    sP[r * L::LDC + i] = dec * qk[a][c];
                    sU[r * L::LDV + i] = br * (sV[r * L::LDV + i] - gam * xs[a][c]);
                    o_acc[a][c] *= gam;
                }
            }
        }
        __syncthreads();

        // ---- phase 2: U = (I + A)^{-1} R ----
        solve_unit_lower<L::LDC, L::LDV>(sA, sU);

        // ---- phase 3: O += (QK^T * L) U, store ----
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
            if (o != nullptr && r < n) {
                Tio *orow = o + (tok0 + (size_t)r * H) * dv + vcol0;
#pragma unroll
                for (int c = 0; c < 4; ++c) orow[tx + 16 * c] = from_f32<Tio>(o_acc[a][c]);
            }
        }
        __syncthreads();  // all reads of U as the intra-chunk operand are done

        // ---- phase 4: U <- diag(exp(g_C - g)) U ----
        for (int idx = tid; idx < kChunk * kSimtDvs; idx += blockDim.x) {
            const int r = idx / kSimtDvs, c = idx % kSimtDvs;
            sU[r * L::LDV + c] *= sDec[r];
        }
        __syncthreads();

        // ---- phase 5: S <- gamma_C S + U~^T K ----
        {
            constexpr int NB = DK / 16;
            float acc[4][NB];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < NB; ++c) acc[a][c] = 0.f;
#pragma unroll 4
            for (int r = 0; r < kChunk; ++r) {
                float ur[4], kr[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) ur[a] = sU[r * L::LDV + ty + 16 * a];
#pragma unroll
                for (int c = 0; c < NB; ++c) kr[c] = sK[r * L::LDK + tx + 16 * c];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < NB; ++c) acc[a][c] = fmaf(ur[a], kr[c], acc[a][c]);
            }
            const float gC = sGam[kChunk - 1];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < NB; ++c) {
                    float *s = &sS[(ty + 16 * a) * L::LDK + tx + 16 * c];
                    *s = fmaf(gC, *s, acc[a][c]);
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
cudaError_t launch_fwd_simt(int B, int T, int H, int dv, const void *q, const void *k,
                            const void *v, const float *la, const float *beta, const float *S0,
                            void *o, float *S_T, cudaStream_t stream,
                            float *S_chunks = nullptr) {
    using L = FwdSimtLayout<DK>;
    auto kern = gdr_fwd_simt_kernel<Tio, DK>;
    cudaError_t err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)L::kBytes);
    if (err != cudaSuccess) return err;
    dim3 grid((unsigned)(B * H) * (unsigned)(dv / kSimtDvs));
    kern<<<grid, kSimtThreads, L::kBytes, stream>>>(
        T, H, dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k),
        static_cast<const Tio *>(v), la, beta, S0, static_cast<Tio *>(o), S_T, S_chunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
