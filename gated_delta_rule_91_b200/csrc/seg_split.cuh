// seg_split.cuh -- splitting one sequence into segments (one per GPU).
//
// For one (b, h) the gated delta rule over a segment maps the incoming state
// affinely, S_out = S_in M + N: N is the segment's final state from S_in = 0
// and M (dk x dk) the product of the per-token factors alpha_t (I - beta_t
// k_t k_t^T) in token order -- in the chunkwise form of the Gated DeltaNet
// review (section 3.7), the product of the chunks' (gamma_C I - W^T K)
// factors.  The readout is affine as well: o_t = S_in (M_<=t q_t) + o_t(0).
// The same rule run with v = 0 from S0 = I (so dv = dk) returns M as its
// final state and q~_t = M_<=t q_t as its outputs.  So a segment takes two
// forward passes (gdr_seg_fwd), an exchange of (M, N) between the segments,
// a sequential combine (gdr_seg_combine) and the correction o += S_in q~
// (gdr_seg_fixup).  The kernels here are the identity initialiser, the
// combine and the correction; all arithmetic is fp32.
#pragma once

#include "common.cuh"

namespace gdr {

constexpr int kSegThreads = 256;

// S[bh] = I (dk x dk) for every (batch, head).
__global__ void __launch_bounds__(kSegThreads) seg_identity_kernel(float *S, int dk, long long n) {
    for (long long i = blockIdx.x * (long long)kSegThreads + threadIdx.x; i < n;
         i += (long long)gridDim.x * kSegThreads) {
        const int e = (int)(i % ((long long)dk * dk));
        S[i] = (e / dk == e % dk) ? 1.f : 0.f;
    }
}

// One block per (batch, head): S = S0 (or 0); for segment j = 0 .. R-1:
// S = S M_j + N_j, writing S_in = S before segment r and S_T = S after the
// last one.  M: [R, B*H, dk, dk]; N: [R, B*H, dv, dk]; S0, S_in, S_T:
// [B*H, dv, dk].  A thread owns DV/16 rows x DK/16 columns of the product
// (rows ty + 16a, columns tx + 16c), read from S and M staged in shared
// memory.
template <int DK, int DV>
__global__ void __launch_bounds__(kSegThreads)
    seg_combine_kernel(int R, int r, int BH, const float *__restrict__ M, const float *__restrict__ N,
                       const float *__restrict__ S0, float *__restrict__ S_in, float *__restrict__ S_T) {
    extern __shared__ __align__(16) float seg_smem[];
    float *sS = seg_smem;            // [DV][DK]
    float *sM = seg_smem + DV * DK;  // [DK][DK]
    constexpr int RA = DV / 16, CA = DK / 16;
    const int bh = blockIdx.x, tx = threadIdx.x % 16, ty = threadIdx.x / 16;
    const size_t sz = (size_t)DV * DK, mz = (size_t)DK * DK;
    for (int i = threadIdx.x; i < DV * DK; i += kSegThreads) sS[i] = S0 ? S0[bh * sz + i] : 0.f;
    __syncthreads();
    if (r == 0 && S_in)
        for (int i = threadIdx.x; i < DV * DK; i += kSegThreads) S_in[bh * sz + i] = sS[i];
    const int last = S_T ? R : r;  // segments whose map is applied
    for (int j = 0; j < last; ++j) {
        const float *Mj = M + ((size_t)j * BH + bh) * mz;
        const float *Nj = N + ((size_t)j * BH + bh) * sz;
        for (int i = threadIdx.x; i < DK * DK / 4; i += kSegThreads)
            reinterpret_cast<float4 *>(sM)[i] = reinterpret_cast<const float4 *>(Mj)[i];
        __syncthreads();
        float acc[RA][CA];
#pragma unroll
        for (int a = 0; a < RA; ++a)
#pragma unroll
            for (int c = 0; c < CA; ++c) acc[a][c] = Nj[(size_t)(ty + 16 * a) * DK + tx + 16 * c];
#pragma unroll 4
        for (int l = 0; l < DK; ++l) {
            float sv[RA], mv[CA];
#pragma unroll
            for (int a = 0; a < RA; ++a) sv[a] = sS[(ty + 16 * a) * DK + l];
#pragma unroll
            for (int c = 0; c < CA; ++c) mv[c] = sM[l * DK + tx + 16 * c];
#pragma unroll
            for (int a = 0; a < RA; ++a)
#pragma unroll
                for (int c = 0; c < CA; ++c) acc[a][c] = fmaf(sv[a], mv[c], acc[a][c]);
        }
        __syncthreads();  // every thread is done reading sS and sM
#pragma unroll
        for (int a = 0; a < RA; ++a)
#pragma unroll
            for (int c = 0; c < CA; ++c) sS[(ty + 16 * a) * DK + tx + 16 * c] = acc[a][c];
        __syncthreads();
        if (j + 1 == r && S_in)
            for (int i = threadIdx.x; i < DV * DK; i += kSegThreads) S_in[bh * sz + i] = sS[i];
    }
    if (S_T)
        for (int i = threadIdx.x; i < DV * DK; i += kSegThreads) S_T[bh * sz + i] = sS[i];
}

// o[b, t, h, :] += S_in[b, h] q~[b, t, h, :] for the tokens of a segment.
// Block (bh, g) keeps S_in^T in shared memory and walks 32-token tiles
// g, g + G, ...; a thread owns 4 tokens (tt + 8a) x DV/32 outputs (ti + 32c).
constexpr int kFixTok = 32;

template <typename Tio, int DK, int DV>
__global__ void __launch_bounds__(kSegThreads)
    seg_fixup_kernel(int T, int H, const Tio *__restrict__ qt, const float *__restrict__ S_in, Tio *__restrict__ o) {
    extern __shared__ __align__(16) float seg_smem[];
    float *sSt = seg_smem;            // [DK][DV]: S_in transposed
    float *sQ = seg_smem + DK * DV;   // [kFixTok][DK]
    constexpr int CO = DV / 32;
    const int head = blockIdx.x, g = blockIdx.y, G = gridDim.y;
    const int b = head / H, h = head % H;
    const int ti = threadIdx.x % 32, tt = threadIdx.x / 32;
    const float *S = S_in + (size_t)head * DV * DK;
    for (int i = threadIdx.x; i < DV * DK; i += kSegThreads) {
        const int col = i / DV, row = i % DV;  // St[col][row] = S[row][col]
        sSt[i] = S[(size_t)row * DK + col];
    }
    const int tiles = (T + kFixTok - 1) / kFixTok;
    for (int tile = g; tile < tiles; tile += G) {
        const int t0 = tile * kFixTok, n = min(kFixTok, T - t0);
        __syncthreads();  // sSt written / previous tile's sQ consumed
        for (int i = threadIdx.x; i < kFixTok * DK; i += kSegThreads) {
            const int t = i / DK, j = i % DK;
            sQ[i] = t < n ? to_f32(qt[(((size_t)b * T + t0 + t) * H + h) * DK + j]) : 0.f;
        }
        __syncthreads();
        float acc[4][CO];
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
            for (int c = 0; c < CO; ++c) acc[a][c] = 0.f;
#pragma unroll 4
        for (int j = 0; j < DK; ++j) {
            float qv[4], sv[CO];
#pragma unroll
            for (int a = 0; a < 4; ++a) qv[a] = sQ[(tt + 8 * a) * DK + j];
#pragma unroll
            for (int c = 0; c < CO; ++c) sv[c] = sSt[j * DV + ti + 32 * c];
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < CO; ++c) acc[a][c] = fmaf(qv[a], sv[c], acc[a][c]);
        }
#pragma unroll
        for (int a = 0; a < 4; ++a) {
            const int t = tt + 8 * a;
            if (t >= n) continue;
            Tio *orow = o + (((size_t)b * T + t0 + t) * H + h) * DV;
#pragma unroll
            for (int c = 0; c < CO; ++c) {
                const int i = ti + 32 * c;
                orow[i] = from_f32<Tio>(to_f32(orow[i]) + acc[a][c]);
            }
        }
    }
}

inline cudaError_t launch_seg_identity(float *S, int BH, int dk, cudaStream_t stream) {
    const long long n = (long long)BH * dk * dk;
    const int grid = (int)std::min<long long>((n + kSegThreads - 1) / kSegThreads, 4096);
    seg_identity_kernel<<<grid, kSegThreads, 0, stream>>>(S, dk, n);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

template <int DK, int DV>
inline cudaError_t launch_seg_combine_t(int R, int r, int BH, const float *M, const float *N, const float *S0,
                                        float *S_in, float *S_T, cudaStream_t stream) {
    const int smem = (DV * DK + DK * DK) * 4;
    cudaError_t e = cudaFuncSetAttribute(seg_combine_kernel<DK, DV>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    seg_combine_kernel<DK, DV><<<BH, kSegThreads, smem, stream>>>(R, r, BH, M, N, S0, S_in, S_T);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

inline cudaError_t launch_seg_combine(int R, int r, int BH, int dk, int dv, const float *M, const float *N,
                                      const float *S0, float *S_in, float *S_T, cudaStream_t stream) {
    if (dk == 128 && dv == 128) return launch_seg_combine_t<128, 128>(R, r, BH, M, N, S0, S_in, S_T, stream);
    if (dk == 128 && dv == 64) return launch_seg_combine_t<128, 64>(R, r, BH, M, N, S0, S_in, S_T, stream);
    if (dk == 64 && dv == 128) return launch_seg_combine_t<64, 128>(R, r, BH, M, N, S0, S_in, S_T, stream);
    return launch_seg_combine_t<64, 64>(R, r, BH, M, N, S0, S_in, S_T, stream);
}

template <typename Tio, int DK, int DV>
inline cudaError_t launch_seg_fixup_t(int B, int T, int H, const void *qt, const float *S_in, void *o,
                                      cudaStream_t stream) {
    const int smem = (DK * DV + kFixTok * DK) * 4;
    auto kern = seg_fixup_kernel<Tio, DK, DV>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int tiles = (T + kFixTok - 1) / kFixTok;
    const int G = std::max(1, std::min(tiles, (2 * sms + B * H - 1) / (B * H)));
    kern<<<dim3(B * H, G), kSegThreads, smem, stream>>>(T, H, static_cast<const Tio *>(qt), S_in,
                                                        static_cast<Tio *>(o));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

template <typename Tio>
inline cudaError_t launch_seg_fixup(int B, int T, int H, int dk, int dv, const void *qt, const float *S_in, void *o,
                                    cudaStream_t stream) {
    if (dk == 128 && dv == 128) return launch_seg_fixup_t<Tio, 128, 128>(B, T, H, qt, S_in, o, stream);
    if (dk == 128 && dv == 64) return launch_seg_fixup_t<Tio, 128, 64>(B, T, H, qt, S_in, o, stream);
    if (dk == 64 && dv == 128) return launch_seg_fixup_t<Tio, 64, 128>(B, T, H, qt, S_in, o, stream);
    return launch_seg_fixup_t<Tio, 64, 64>(B, T, H, qt, S_in, o, stream);
}

}  // namespace gdr
