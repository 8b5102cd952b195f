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
#include "sm100.cuh"
#include "fwd_tc.cuh"  // make_token_map

namespace gdr {

constexpr int kSegThreads = 256;

// Four consecutive elements of a row (16-byte aligned for fp32, 8 for bf16).
__device__ __forceinline__ void ld_row4(const float *p, float *v) {
    const float4 f = *reinterpret_cast<const float4 *>(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
__device__ __forceinline__ void ld_row4(const __nv_bfloat16 *p, float *v) {
    const float4 f = load4(p);
    v[0] = f.x; v[1] = f.y; v[2] = f.z; v[3] = f.w;
}
__device__ __forceinline__ void st_row4(float *p, const float *v) {
    *reinterpret_cast<float4 *>(p) = make_float4(v[0], v[1], v[2], v[3]);
}
__device__ __forceinline__ void st_row4(__nv_bfloat16 *p, const float *v) {
    __nv_bfloat162 a = __floats2bfloat162_rn(v[0], v[1]), b = __floats2bfloat162_rn(v[2], v[3]);
    uint2 raw;
    raw.x = *reinterpret_cast<uint32_t *>(&a);
    raw.y = *reinterpret_cast<uint32_t *>(&b);
    *reinterpret_cast<uint2 *>(p) = raw;
}

// S[bh] = I (dk x dk) for every (batch, head).
__global__ void __launch_bounds__(kSegThreads) seg_identity_kernel(float *S, int dk, long long n) {
    for (long long i = blockIdx.x * (long long)kSegThreads + threadIdx.x; i < n;
         i += (long long)gridDim.x * kSegThreads) {
        const int e = (int)(i % ((long long)dk * dk));
        S[i] = (e / dk == e % dk) ? 1.f : 0.f;
    }
}

// The combine.  S = S0 (or 0); for segment j = 0 .. R-1: S = S M_j + N_j,
// writing S_in = S before segment r and S_T = S after the last one.  Rows of
// S are independent, so block (bh, rb) carries rows [32 rb, 32 rb + 32) of
// one (batch, head) through all the steps, staging M_j in shared memory.
// M: [R, B*H, dk, dk]; N: [R, B*H, dv, dk]; S0, S_in, S_T: [B*H, dv, dk].
// A thread owns RPT rows (2 for dk = 128, 1 for dk = 64) x 8 columns (two
// float4 of M per k step).
constexpr int kCombRows = 32;

template <int DK>
__global__ void __launch_bounds__(kSegThreads)
    seg_combine_kernel(int R, int r, int BH, int DV, const float *__restrict__ M, const float *__restrict__ N,
                       const float *__restrict__ S0, float *__restrict__ S_in, float *__restrict__ S_T) {
    extern __shared__ __align__(16) float seg_smem[];
    float *sM = seg_smem;             // [DK][DK]
    float *sS = seg_smem + DK * DK;   // [kCombRows][DK]
    constexpr int CG = DK / 8;               // column groups (8 columns each)
    constexpr int RG = kSegThreads / CG;     // row groups
    constexpr int RPT = kCombRows / RG;      // rows per thread
    static_assert(RPT * RG == kCombRows && RPT >= 1, "row split");
    const int bh = blockIdx.x, row0 = blockIdx.y * kCombRows;
    const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
    // columns of this thread: 4 cg .. 4 cg + 3 and DK/2 + 4 cg .. + 3
    const int c0 = 4 * cg, c1 = DK / 2 + 4 * cg;
    const size_t sz = (size_t)DV * DK, mz = (size_t)DK * DK;
    for (int i = threadIdx.x; i < kCombRows * DK; i += kSegThreads)
        sS[i] = S0 ? S0[bh * sz + (size_t)row0 * DK + i] : 0.f;
    __syncthreads();
    auto write_rows = [&](float *dst) {
        for (int i = threadIdx.x; i < kCombRows * DK; i += kSegThreads) dst[bh * sz + (size_t)row0 * DK + i] = sS[i];
    };
    if (r == 0 && S_in) write_rows(S_in);
    const int last = S_T ? R : r;  // segments whose map is applied
    for (int j = 0; j < last; ++j) {
        const float *Mj = M + ((size_t)j * BH + bh) * mz;
        const float *Nj = N + ((size_t)j * BH + bh) * sz + (size_t)row0 * DK;
        for (int i = threadIdx.x; i < DK * DK / 4; i += kSegThreads)
            reinterpret_cast<float4 *>(sM)[i] = reinterpret_cast<const float4 *>(Mj)[i];
        float acc[RPT][8];
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            const float *nr = Nj + (size_t)(rg + RG * a) * DK;
            const float4 n0 = *reinterpret_cast<const float4 *>(nr + c0);
            const float4 n1 = *reinterpret_cast<const float4 *>(nr + c1);
            acc[a][0] = n0.x; acc[a][1] = n0.y; acc[a][2] = n0.z; acc[a][3] = n0.w;
            acc[a][4] = n1.x; acc[a][5] = n1.y; acc[a][6] = n1.z; acc[a][7] = n1.w;
        }
        __syncthreads();  // sM staged
#pragma unroll 4
        for (int l = 0; l < DK; ++l) {
            const float4 m0 = *reinterpret_cast<const float4 *>(sM + l * DK + c0);
            const float4 m1 = *reinterpret_cast<const float4 *>(sM + l * DK + c1);
            const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
            for (int a = 0; a < RPT; ++a) {
                const float sv = sS[(rg + RG * a) * DK + l];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(sv, mv[c], acc[a][c]);
            }
        }
        __syncthreads();  // every thread is done reading sS and sM
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            float *sr = sS + (rg + RG * a) * DK;
            *reinterpret_cast<float4 *>(sr + c0) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
            *reinterpret_cast<float4 *>(sr + c1) = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
        }
        __syncthreads();
        if (j + 1 == r && S_in) write_rows(S_in);
    }
    if (S_T) write_rows(S_T);
}

// The same combine for R segments of every batch on one GPU (a sequence
// viewed as [B*R, T/R, H, d]): M, N: [B*R, H, ...] with segment r of batch b
// at head index (b R + r) H + h.  Block (b*H + h, rb) walks r = 0 .. R-1,
// writing S_in of every segment ([B*R, H, dv, dk]) and the final state S_T
// ([B, H, dv, dk], may be null).  With S0 null the first segment's M is
// never read (S is zero there).
template <int DK>
__global__ void __launch_bounds__(kSegThreads)
    seg_scan_kernel(int R, int H, int DV, const float *__restrict__ M, const float *__restrict__ N,
                    const float *__restrict__ S0, float *__restrict__ S_in, float *__restrict__ S_T) {
    extern __shared__ __align__(16) float seg_smem[];
    float *sM = seg_smem;             // [DK][DK]
    float *sS = seg_smem + DK * DK;   // [kCombRows][DK]
    constexpr int CG = DK / 8, RG = kSegThreads / CG, RPT = kCombRows / RG;
    const int bh = blockIdx.x, b = bh / H, h = bh % H, row0 = blockIdx.y * kCombRows;
    const int cg = threadIdx.x % CG, rg = threadIdx.x / CG;
    const int c0 = 4 * cg, c1 = DK / 2 + 4 * cg;
    const size_t sz = (size_t)DV * DK, mz = (size_t)DK * DK;
    for (int i = threadIdx.x; i < kCombRows * DK; i += kSegThreads)
        sS[i] = S0 ? S0[bh * sz + (size_t)row0 * DK + i] : 0.f;
    __syncthreads();
    for (int j = 0; j < R; ++j) {
        const size_t seg = ((size_t)b * R + j) * H + h;
        for (int i = threadIdx.x; i < kCombRows * DK; i += kSegThreads) S_in[seg * sz + (size_t)row0 * DK + i] = sS[i];
        if (j + 1 == R && S_T == nullptr) break;
        if (j == 0 && S0 == nullptr) {  // S = 0: the map of segment 0 is N_0 alone (M_0 is not read)
            __syncthreads();
            for (int i = threadIdx.x; i < kCombRows * DK; i += kSegThreads)
                sS[i] = N[seg * sz + (size_t)row0 * DK + i];
            __syncthreads();
            continue;
        }
        const float *Mj = M + seg * mz;
        const float *Nj = N + seg * sz + (size_t)row0 * DK;
        for (int i = threadIdx.x; i < DK * DK / 4; i += kSegThreads)
            reinterpret_cast<float4 *>(sM)[i] = reinterpret_cast<const float4 *>(Mj)[i];
        float acc[RPT][8];
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            const float *nr = Nj + (size_t)(rg + RG * a) * DK;
            const float4 n0 = *reinterpret_cast<const float4 *>(nr + c0);
            const float4 n1 = *reinterpret_cast<const float4 *>(nr + c1);
            acc[a][0] = n0.x; acc[a][1] = n0.y; acc[a][2] = n0.z; acc[a][3] = n0.w;
            acc[a][4] = n1.x; acc[a][5] = n1.y; acc[a][6] = n1.z; acc[a][7] = n1.w;
        }
        __syncthreads();  // sM staged; sS copied out
#pragma unroll 4
        for (int l = 0; l < DK; ++l) {
            const float4 m0 = *reinterpret_cast<const float4 *>(sM + l * DK + c0);
            const float4 m1 = *reinterpret_cast<const float4 *>(sM + l * DK + c1);
            const float mv[8] = {m0.x, m0.y, m0.z, m0.w, m1.x, m1.y, m1.z, m1.w};
#pragma unroll
            for (int a = 0; a < RPT; ++a) {
                const float sv = sS[(rg + RG * a) * DK + l];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(sv, mv[c], acc[a][c]);
            }
        }
        __syncthreads();
#pragma unroll
        for (int a = 0; a < RPT; ++a) {
            float *sr = sS + (rg + RG * a) * DK;
            *reinterpret_cast<float4 *>(sr + c0) = make_float4(acc[a][0], acc[a][1], acc[a][2], acc[a][3]);
            *reinterpret_cast<float4 *>(sr + c1) = make_float4(acc[a][4], acc[a][5], acc[a][6], acc[a][7]);
        }
        __syncthreads();
    }
    if (S_T)
        for (int i = threadIdx.x; i < kCombRows * DK; i += kSegThreads) S_T[bh * sz + (size_t)row0 * DK + i] = sS[i];
}

inline cudaError_t launch_seg_scan(int B, int R, int H, int dk, int dv, const float *M, const float *N,
                                   const float *S0, float *S_in, float *S_T, cudaStream_t stream) {
    auto run = [&](auto kern, int DK) -> cudaError_t {
        const int smem = (DK * DK + kCombRows * DK) * 4;
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        kern<<<dim3(B * H, dv / kCombRows), kSegThreads, smem, stream>>>(R, H, dv, M, N, S0, S_in, S_T);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cudaGetLastError();
    };
    return dk == 128 ? run(seg_scan_kernel<128>, 128) : run(seg_scan_kernel<64>, 64);
}

// o[b, t, h, :] += S_in[b, h] q~[b, t, h, :] for the tokens of a segment.
// Block (bh, g) keeps S_in^T in shared memory and walks 64-token tiles
// g, g + G, ...; a thread owns 4 tokens (tg + 16a) x 8 outputs (4 og .. +3
// and DV/2 + 4 og .. +3), read as float4 rows of S_in^T.  q~ rows are padded
// by one float so the token groups of a warp hit different banks.
constexpr int kFixTok = 64;

template <typename Tio, int DK, int DV>
__global__ void __launch_bounds__(kSegThreads)
    seg_fixup_kernel(int T, int H, const Tio *__restrict__ qt, const float *__restrict__ S_in, Tio *__restrict__ o) {
    extern __shared__ __align__(16) float seg_smem[];
    constexpr int LDQ = DK + 1;
    float *sSt = seg_smem;            // [DK][DV]: S_in transposed
    float *sQ = seg_smem + DK * DV;   // [kFixTok][LDQ]
    constexpr int OG = DV / 8, TG = kSegThreads / OG, TA = kFixTok / TG;  // TA tokens per thread
    const int head = blockIdx.x, g = blockIdx.y, G = gridDim.y;
    const int b = head / H, h = head % H;
    const int og = threadIdx.x % OG, tg = threadIdx.x / OG;
    const int c0 = 4 * og, c1 = DV / 2 + 4 * og;
    const float *S = S_in + (size_t)head * DV * DK;
    for (int i = threadIdx.x; i < DV * DK; i += kSegThreads) {
        const int col = i / DV, row = i % DV;  // St[col][row] = S[row][col]
        sSt[i] = S[(size_t)row * DK + col];
    }
    const int tiles = (T + kFixTok - 1) / kFixTok;
    for (int tile = g; tile < tiles; tile += G) {
        const int t0 = tile * kFixTok, n = min(kFixTok, T - t0);
        __syncthreads();  // sSt written / previous tile's sQ consumed
        for (int i = threadIdx.x; i < kFixTok * DK / 8; i += kSegThreads) {  // 8 elements per piece
            const int t = i / (DK / 8), j8 = (i % (DK / 8)) * 8;
            float v[8];
            if (t < n)
                load8(qt + (((size_t)b * T + t0 + t) * H + h) * DK + j8, v);
            else
#pragma unroll
                for (int e = 0; e < 8; ++e) v[e] = 0.f;
#pragma unroll
            for (int e = 0; e < 8; ++e) sQ[t * LDQ + j8 + e] = v[e];
        }
        __syncthreads();
        float acc[TA][8];
#pragma unroll
        for (int a = 0; a < TA; ++a)
#pragma unroll
            for (int c = 0; c < 8; ++c) acc[a][c] = 0.f;
#pragma unroll 4
        for (int j = 0; j < DK; ++j) {
            const float4 s0 = *reinterpret_cast<const float4 *>(sSt + j * DV + c0);
            const float4 s1 = *reinterpret_cast<const float4 *>(sSt + j * DV + c1);
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int a = 0; a < TA; ++a) {
                const float qv = sQ[(tg + TG * a) * LDQ + j];
#pragma unroll
                for (int c = 0; c < 8; ++c) acc[a][c] = fmaf(qv, sv[c], acc[a][c]);
            }
        }
#pragma unroll
        for (int a = 0; a < TA; ++a) {
            const int t = tg + TG * a;
            if (t >= n) continue;
            Tio *orow = o + (((size_t)b * T + t0 + t) * H + h) * DV;
#pragma unroll
            for (int half = 0; half < 2; ++half) {
                const int cc = half ? c1 : c0;
                float cur[4];
                ld_row4(orow + cc, cur);
#pragma unroll
                for (int e = 0; e < 4; ++e) cur[e] += acc[a][4 * half + e];
                st_row4(orow + cc, cur);
            }
        }
    }
}

// Tensor-core correction for bf16 with dk = dv = 128: per 128-token tile,
// D[t, i] = sum_j q~[t, j] S_in[i, j] is one M128 N128 K128 tcgen05 product
// (A = the q~ tile, B = S_in as bf16, both K-major with 128-byte swizzle, D in
// TMEM); the epilogue adds D into the o tile staged by TMA and stores it back
// with TMA.  Two stages: the next tile's loads fly while this one is
// multiplied and finished.  128 threads: thread t of the epilogue owns token
// row t of the tile (its warp's TMEM lane quarter).
//
// The heads are the segments r0 .. R-1 of every batch of a [B*R, T, H, 128]
// view (a plain [B, T, H, 128] tensor is R = 1, r0 = 0): block (x, g) takes
// batch x / ((R - r0) H), segment r0 + (x / H) % (R - r0), head x % H, and
// walks tiles g, g + G, ...
constexpr int kFixTcThreads = 128;
struct FixTcLayout {
    static constexpr int S = 0;           // S_in bf16: 2 K-halves x [128][64], 16 KB each
    static constexpr int ST0 = 32768;     // stage s at ST0 + s * 65536: q~ tile (2 K-halves x [128][64]),
    static constexpr int QOFF = 0;        //   then the o tile (2 channel halves x 2 token halves x [64][64])
    static constexpr int OOFF = 32768;
    static constexpr int BAR = ST0 + 2 * 65536;  // 2 load barriers, 1 MMA barrier, TMEM address
    static constexpr int kBytes = BAR + 64;
    static constexpr int kAlloc = kBytes + 1024;  // slack to align the base to 1024
};

__global__ void __launch_bounds__(kFixTcThreads)
    seg_fixup_tc_kernel(const __grid_constant__ CUtensorMap tm_qt, const __grid_constant__ CUtensorMap tm_o, int T,
                        int H, int R, int r0, const float *__restrict__ S_in) {
    using namespace sm100;
    using L = FixTcLayout;
    extern __shared__ uint8_t fix_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(fix_raw) + 1023) & ~uintptr_t(1023));
    uint64_t *bar_tma = reinterpret_cast<uint64_t *>(sm + L::BAR);  // [2]
    uint64_t *bar_mma = bar_tma + 2;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bar_tma + 3);
    const int nseg = R - r0;
    const int b = blockIdx.x / (nseg * H), r = r0 + (blockIdx.x / H) % nseg, h = blockIdx.x % H;
    const int bs = b * R + r;  // batch index in the [B*R, T, H, 128] view
    const int g = blockIdx.y, G = gridDim.y;
    const int tid = threadIdx.x, warp = tid >> 5;
    if (tid == 0) {
        mbar_init(&bar_tma[0], 1);
        mbar_init(&bar_tma[1], 1);
        mbar_init(bar_mma, 1);
        fence_mbar_init();
    }
    if (warp == 0) tmem_alloc(tmem_slot, 128);
    // S_in (fp32 [128][128]) -> bf16 B operand: row i, column j in K-half j / 64
    const float *S = S_in + ((size_t)bs * H + h) * 128 * 128;
    for (int p = tid; p < 128 * 64; p += kFixTcThreads) {
        const int i = p / 64, j = (p % 64) * 2;
        const float2 v = *reinterpret_cast<const float2 *>(S + (size_t)i * 128 + j);
        st_sw_bf16x2(sm + L::S + (j >> 6) * 16384, i, j & 63, v.x, v.y);
    }
    fence_async_smem();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    const uint32_t tl = *tmem_slot;
    const int tiles = (T + 127) / 128;
    auto issue_loads = [&](int tile, int st) {  // one thread
        uint8_t *stage = sm + L::ST0 + st * 65536;
        const int t0 = tile * 128;
        mbar_expect_tx(&bar_tma[st], 65536);
#pragma unroll
        for (int kh = 0; kh < 2; ++kh)
#pragma unroll
            for (int th = 0; th < 2; ++th) {
                tma_load_4d(stage + L::QOFF + kh * 16384 + th * 8192, &tm_qt, &bar_tma[st], kh * 64, h, t0 + th * 64, bs);
                tma_load_4d(stage + L::OOFF + kh * 16384 + th * 8192, &tm_o, &bar_tma[st], kh * 64, h, t0 + th * 64, bs);
            }
    };
    if (tid == 0 && g < tiles) issue_loads(g, 0);
    bool ok = true;
    int k = 0;
    for (int tile = g; tile < tiles; tile += G, ++k) {
        const int st = k & 1;
        uint8_t *stage = sm + L::ST0 + st * 65536;
        if (!__syncthreads_and(mbar_wait(&bar_tma[st], (uint32_t)(k >> 1) & 1u))) {  // the block agrees
            ok = false;
            break;
        }
        if (tid == 0) {
            tc_after_sync();
            const uint32_t sq = smem_u32(stage + L::QOFF), ss = smem_u32(sm + L::S);
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tl, smem_desc_sw128(sq + kh * 16384 + kk * 32, 16, 1024),
                             smem_desc_sw128(ss + kh * 16384 + kk * 32, 16, 1024), idesc_bf16(128, 128, false, false),
                             (kh | kk) != 0);
            mma_commit(bar_mma);
            // the next tile into the other stage, once its previous o tile has
            // been read out by the TMA store
            if (tile + G < tiles) {
                bulk_wait_read_all();
                issue_loads(tile + G, st ^ 1);
            }
        }
        if (!__syncthreads_and(mbar_wait(bar_mma, (uint32_t)k & 1u))) {
            ok = false;
            break;
        }
        tc_after_sync();
        // epilogue: row t of the tile (token t0 + t) += D[t, :]
        const int t = tid, th = t >> 6, rr = t & 63;
#pragma unroll
        for (int c32 = 0; c32 < 4; ++c32) {
            float d[32];
            tmem_ld32(tl + ((uint32_t)(warp * 32) << 16) + c32 * 32, d);
            uint8_t *tileo = stage + L::OOFF + (c32 >> 1) * 16384 + th * 8192;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                const int chunk = (c32 & 1) * 4 + q;  // 16-byte chunk of the 128-byte row
                uint4 *pc = reinterpret_cast<uint4 *>(tileo + sw128_offset(rr, chunk));
                uint4 raw = *pc;
                __nv_bfloat162 *hv = reinterpret_cast<__nv_bfloat162 *>(&raw);
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 f = __bfloat1622float2(hv[e]);
                    hv[e] = __floats2bfloat162_rn(f.x + d[q * 8 + 2 * e], f.y + d[q * 8 + 2 * e + 1]);
                }
                *pc = raw;
            }
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();  // o tile complete; TMEM free for the next product
        if (tid == 0) {
            const int t0 = tile * 128;
#pragma unroll
            for (int kh = 0; kh < 2; ++kh)
#pragma unroll
                for (int th2 = 0; th2 < 2; ++th2)
                    tma_store_4d(&tm_o, stage + L::OOFF + kh * 16384 + th2 * 8192, kh * 64, h, t0 + th2 * 64, bs);
            bulk_commit();
        }
    }
    if (!ok) record_status(GDR_ERR_TIMEOUT);
    if (tid == 0) bulk_wait_all();
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    if (warp == 0) tmem_dealloc(tl, 128);
}

// o [B*R, T, H, 128] += S_in q~ for the segments r0 .. R-1 of every batch
// (R = 1, r0 = 0: a plain [B, T, H, 128] tensor).
inline cudaError_t launch_seg_fixup_tc(int B, int T, int H, const void *qt, const float *S_in, void *o,
                                       cudaStream_t stream, int R = 1, int r0 = 0) {
    CUtensorMap mq, mo;
    if (!make_token_map(&mq, qt, B * R, T, H, 128) || !make_token_map(&mo, o, B * R, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t e = cudaFuncSetAttribute(seg_fixup_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         FixTcLayout::kAlloc);
    if (e != cudaSuccess) return e;
    int dev = 0, sms = 148;
    if (cudaGetDevice(&dev) == cudaSuccess) cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int heads = B * (R - r0) * H;
    const int tiles = (T + 127) / 128;
    // one block per SM (its shared memory): G blocks per head in one wave
    const int G = std::max(1, std::min(tiles, sms / heads));
    seg_fixup_tc_kernel<<<dim3(heads, G), kFixTcThreads, FixTcLayout::kAlloc, stream>>>(mq, mo, T, H, R, r0, S_in);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

inline cudaError_t launch_seg_identity(float *S, int BH, int dk, cudaStream_t stream) {
    const long long n = (long long)BH * dk * dk;
    const int grid = (int)std::min<long long>((n + kSegThreads - 1) / kSegThreads, 4096);
    seg_identity_kernel<<<grid, kSegThreads, 0, stream>>>(S, dk, n);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

template <int DK>
inline cudaError_t launch_seg_combine_t(int R, int r, int BH, int dv, const float *M, const float *N, const float *S0,
                                        float *S_in, float *S_T, cudaStream_t stream) {
    const int smem = (DK * DK + kCombRows * DK) * 4;
    cudaError_t e = cudaFuncSetAttribute(seg_combine_kernel<DK>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    if (e != cudaSuccess) return e;
    seg_combine_kernel<DK><<<dim3(BH, dv / kCombRows), kSegThreads, smem, stream>>>(R, r, BH, dv, M, N, S0, S_in, S_T);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

inline cudaError_t launch_seg_combine(int R, int r, int BH, int dk, int dv, const float *M, const float *N,
                                      const float *S0, float *S_in, float *S_T, cudaStream_t stream) {
    return dk == 128 ? launch_seg_combine_t<128>(R, r, BH, dv, M, N, S0, S_in, S_T, stream)
                     : launch_seg_combine_t<64>(R, r, BH, dv, M, N, S0, S_in, S_T, stream);
}

template <typename Tio, int DK, int DV>
inline cudaError_t launch_seg_fixup_t(int B, int T, int H, const void *qt, const float *S_in, void *o,
                                      cudaStream_t stream) {
    const int smem = (DK * DV + kFixTok * (DK + 1)) * 4;
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
