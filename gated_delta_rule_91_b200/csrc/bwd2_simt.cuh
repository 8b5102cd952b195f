// bwd2_simt.cuh -- chunkwise backward of Gated DeltaNet-2 on CUDA cores (fp32
// arithmetic; fp32 or bf16 q/k/v/dO).
//
// The pages give no backward; this is the chain rule applied to the chunk
// map of the Gated Delta Rule-2 forward ("Gated DeltaNet-2: Decoupling Erase
// and Write in Linear Attention", agihunt.info/papers/2605.22791, the Gated
// Delta Rule-2 paragraph; the chunk form is restated in gdr2_simt.cuh).  Per
// chunk, with G the per-channel cumulative log decay, E = exp(G),
//     KBE = K*B*E, QE = Q*E, KiE = K/E, Kt = K*exp(G_C - G) = KiE Diag(E_C),
//     A = strictLower(KBE KiE^T), P = inclLower(QE KiE^T), T = (I + A)^{-1},
//     R = W*V - KBE S^T, U = T R, O = QE S^T + P U, S' = S Diag(E_C) + U^T Kt,
// and D = dL/dS', dO:
//     dU = Kt D^T + P^T dO          dR = T^T dU          dA = -dR U^T (i < r)
//     dP = dO U^T (i <= r)          dV = W*dR            dW = V*dR
//     dKBE = -dR S + dA KiE         dQE = dO S + dP KiE
//     dKiE = dA^T KBE + dP^T QE + (U D) Diag(E_C)
//     dS = D Diag(E_C) + dO^T QE - dR^T KBE            (D of the previous chunk)
//     dE_C = colsum(S * D) + colsum((U D) * KiE)
// then per element dK = dKBE B E + dKiE / E, dB = dKBE K E, dQ = dQE E,
// dG = dKBE KBE + dQE QE - dKiE KiE, plus E_C dE_C on the chunk's last token,
// and dlog alpha = the in-chunk suffix sums of dG per channel.
//
// One CTA owns one (b, h) and a slice of kBwd2Dvs state rows and walks the
// chunks from last to first.  dV, dW and dS are slice-local; dKBE, dQE,
// dKiE and dE_C are sums over slices, written per slice and summed in a
// fixed order by gdr2_bwd_reduce_kernel, which also applies the per-element
// chain rule (deterministic, no atomics).  A chunk in which some channel
// decays by more than e^80 (where K/E would overflow) is walked token by
// token instead, with the step's own reverse mode (gdr2_chunk_reverse_exact);
// its per-token partials are summed by the same reduce kernel without the
// E factors.
//
// For bf16 with dk = dv = 128, launch_bwd2_simt runs another sequence: the
// cluster recompute (which also keeps every chunk's T and P), the
// tensor-core dS pass (bwd2_ds.cuh, every chunk's D), and one tensor-core
// CTA per chunk for all of its gradients (bwd2_grad_tc.cuh).  Only the
// chunks that one lists (decay past e^20) come here: gdr2_bwd_simt_list_kernel
// runs this reverse per (slice, listed chunk) from the stored D, and the
// chunk kernel of bwd2_tc.cuh sums their slices.
#pragma once
#include "common.cuh"
#include "bwd_simt.cuh"
#include "gdr2_simt.cuh"
#include "fwd2_tc.cuh"
#include "fwd2_tc2.cuh"
#include "bwd2_tc.cuh"
#include "bwd2_ds.cuh"
#include "bwd2_grad_tc.cuh"
#include <type_traits>

namespace gdr {

constexpr int kBwd2Dvs = 32;  // state rows per CTA

template <int DK>
struct Bwd2Layout {
    static constexpr int C = kChunk;
    static constexpr int LDK = DK + 1;
    static constexpr int LDV = kBwd2Dvs + 1;
    static constexpr int LDC = C + 1;
    static constexpr int oKB = 0;                    // K*B*E      [C][LDK]
    static constexpr int oQE = oKB + C * LDK;        // Q*E        [C][LDK]
    static constexpr int oKI = oQE + C * LDK;        // K/E        [C][LDK]
    static constexpr int oG = oKI + C * LDK;         // log alpha [C][LDK]; later dP, dA [C][LDC] each
    static constexpr int kGFloats = C * LDK > 2 * C * LDC ? C * LDK : 2 * C * LDC;
    static constexpr int oS = oG + kGFloats;         // entry state slice [kBwd2Dvs][LDK]
    static constexpr int oD = oS + kBwd2Dvs * LDK;   // dL/dS' slice      [kBwd2Dvs][LDK]
    static constexpr int odO = oD + kBwd2Dvs * LDK;  // [C][LDV] each below
    static constexpr int oU = odO + C * LDV;         // R, then U
    static constexpr int odR = oU + C * LDV;         // dU, then dR
    static constexpr int oA = odR + C * LDV;         // [C][LDC] each below
    static constexpr int oP = oA + C * LDC;
    static constexpr int oVec = oP + C * LDC;        // E_C [DK], ones [C], flag
    static constexpr int kFloats = oVec + DK + C + 4;
    static constexpr size_t kBytes = (size_t)kFloats * sizeof(float);
    static_assert(kBytes <= 232448, "shared memory budget");
};

// Reverse of one chunk for this CTA's slice of kBwd2Dvs state rows, token by
// token, for a chunk whose factored operands would overflow.  Per token, with
// S = S_{t-1}, P = S Diag(alpha), e = w*v - P(b*k) (so S_t = P + e k^T) and
// G = dL/dS_t + do q^T, the step's reverse mode is
//     gk = G k,  dv = w * gk,  dw = v * gk,  dL/dS_{t-1} = (G - gk (b*k)^T) Diag(alpha)
// and the key-channel gradients are sums over the state rows:
//     dq = S_t^T do,  dk = G^T e - b * X,  db = -k * X,
//     dlog alpha_j = sum_i P_ij G_ij - b_j k_j X_j,   X = P^T gk.
// This CTA writes its rows' dv, dw and its slice's partial sums of S_t^T do,
// X, G^T e and sum_i P_ij G_ij per token; the reduce kernel adds the slices.
// The states S_{t-1} of an 8-token block are recomputed from the chunk's entry
// state (blocks from last to first) into `st` [8][kBwd2Dvs][DK]; D (dL/dS of
// the slice) stays in registers.  Thread layout: row = tid / 8 of the slice,
// DK / 8 channels from (tid % 8) * DK / 8; row dot products reduce over the
// 8 lanes that share a row.
template <typename Tio, int DK>
__device__ void gdr2_chunk_reverse_exact(int n, size_t tok0, int H, int dv, int vcol0, const Tio *__restrict__ q,
                                         const Tio *__restrict__ k, const Tio *__restrict__ v,
                                         const float *__restrict__ log_alpha, const float *__restrict__ bgate,
                                         const float *__restrict__ wgate, const Tio *__restrict__ dO, float *st,
                                         float *red, const float *sS, float *sD, Tio *__restrict__ dv_out,
                                         float *__restrict__ dw_out, float *__restrict__ part_qe,
                                         float *__restrict__ part_kb, float *__restrict__ part_ki,
                                         float *__restrict__ part_x, size_t pslice) {
    constexpr int JW = DK / 8, LDK = DK + 1, R = kBwd2Dvs;
    static_assert(R * 8 == kSimtThreads, "one row of the slice per 8 threads");
    const int tid = threadIdx.x, row = tid >> 3, j0 = (tid & 7) * JW;
    auto rowsum = [](float x) {
        x += __shfl_xor_sync(0xffffffffu, x, 1);
        x += __shfl_xor_sync(0xffffffffu, x, 2);
        x += __shfl_xor_sync(0xffffffffu, x, 4);
        return x;
    };
    auto ld = [&](const float *p, size_t t, float *out) {  // one token's JW key channels
        const float *src = p + (tok0 + t * H) * DK + j0;
#pragma unroll
        for (int jj = 0; jj < JW; ++jj) out[jj] = src[jj];
    };
    auto ldt = [&](const Tio *p, size_t t, float *out) {
        const Tio *src = p + (tok0 + t * H) * DK + j0;
#pragma unroll
        for (int jj = 0; jj < JW; ++jj) out[jj] = to_f32(src[jj]);
    };
    float d[JW];
#pragma unroll
    for (int jj = 0; jj < JW; ++jj) d[jj] = sD[row * LDK + j0 + jj];
    const int nblk = (n + 7) / 8;
#pragma unroll 1
    for (int blk = nblk - 1; blk >= 0; --blk) {
        const int ts = blk * 8, te = min(n, ts + 8);
        {   // S_{t-1} for t = ts .. te-1, by the forward from the chunk's entry state
            float s[JW];
#pragma unroll
            for (int jj = 0; jj < JW; ++jj) s[jj] = sS[row * LDK + j0 + jj];
#pragma unroll 1
            for (int t = 0; t < te; ++t) {
                if (t >= ts) {
#pragma unroll
                    for (int jj = 0; jj < JW; ++jj) st[((t - ts) * R + row) * DK + j0 + jj] = s[jj];
                }
                if (t + 1 >= te) break;
                float la[JW], bb[JW], kk[JW];
                ld(log_alpha, t, la);
                ld(bgate, t, bb);
                ldt(k, t, kk);
                float r = 0.f;
#pragma unroll
                for (int jj = 0; jj < JW; ++jj) {
                    s[jj] *= expf(la[jj]);
                    r = fmaf(s[jj], bb[jj] * kk[jj], r);
                }
                r = rowsum(r);
                const size_t vo = (tok0 + (size_t)t * H) * dv + vcol0 + row;
                const float e = wgate[vo] * to_f32(v[vo]) - r;
#pragma unroll
                for (int jj = 0; jj < JW; ++jj) s[jj] = fmaf(e, kk[jj], s[jj]);
            }
        }
        __syncthreads();
#pragma unroll 1
        for (int t = te - 1; t >= ts; --t) {
            float la[JW], bb[JW], kk[JW], qq[JW], p[JW], g[JW];
            ld(log_alpha, t, la);
            ld(bgate, t, bb);
            ldt(k, t, kk);
            ldt(q, t, qq);
            const size_t vo = (tok0 + (size_t)t * H) * dv + vcol0 + row;
            const float wv = wgate[vo], vv = to_f32(v[vo]), dov = to_f32(dO[vo]);
            float r = 0.f, gk = 0.f;
#pragma unroll
            for (int jj = 0; jj < JW; ++jj) {
                la[jj] = expf(la[jj]);  // alpha
                p[jj] = st[((t - ts) * R + row) * DK + j0 + jj] * la[jj];
                r = fmaf(p[jj], bb[jj] * kk[jj], r);
                g[jj] = fmaf(dov, qq[jj], d[jj]);
                gk = fmaf(g[jj], kk[jj], gk);
            }
            r = rowsum(r);
            gk = rowsum(gk);
            const float e = wv * vv - r;
            if ((tid & 7) == 0) {
                dv_out[vo] = from_f32<Tio>(wv * gk);
                dw_out[vo] = vv * gk;
            }
            // the four row sums of this token, two at a time through `red` [2][R][DK]
            const size_t prow = pslice * DK + (tok0 + (size_t)t * H) * DK;
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                for (int jj = 0; jj < JW; ++jj) {
                    const float st_ = fmaf(e, kk[jj], p[jj]);  // S_t
                    red[row * DK + j0 + jj] = pass == 0 ? st_ * dov : g[jj] * e;
                    red[(R + row) * DK + j0 + jj] = pass == 0 ? p[jj] * gk : p[jj] * g[jj];
                }
                __syncthreads();
                for (int c = tid; c < 2 * DK; c += kSimtThreads) {
                    const int which = c / DK, j = c % DK;
                    float acc = 0.f;
                    for (int i = 0; i < R; ++i) acc += red[(which * R + i) * DK + j];
                    float *dst = pass == 0 ? (which == 0 ? part_qe : part_ki) : (which == 0 ? part_kb : part_x);
                    dst[prow + j] = acc;
                }
                __syncthreads();
            }
#pragma unroll
            for (int jj = 0; jj < JW; ++jj) d[jj] = (g[jj] - gk * bb[jj] * kk[jj]) * la[jj];
        }
    }
#pragma unroll
    for (int jj = 0; jj < JW; ++jj) sD[row * LDK + j0 + jj] = d[jj];
}

// The reverse of one (b*H + h, slice of value rows) over its chunks, or over
// the one chunk ch_sel when D_chunks (every chunk's exit-state gradient, from
// the tensor-core dS pass) is given.
template <typename Tio, int DK>
__device__ __forceinline__ void gdr2_bwd_simt_body(
    int T, int H, int dv, const Tio *__restrict__ q, const Tio *__restrict__ k, const Tio *__restrict__ v,
    const float *__restrict__ log_alpha, const float *__restrict__ bgate, const float *__restrict__ wgate,
    const Tio *__restrict__ dO, const float *__restrict__ dS_T, const float *__restrict__ S_chunks,
    Tio *__restrict__ dv_out, float *__restrict__ dw_out, float *__restrict__ dS0, float *__restrict__ part_kb,
    float *__restrict__ part_qe, float *__restrict__ part_ki, float *__restrict__ part_ec,
    float *__restrict__ part_x, int *__restrict__ exact_flags, float *__restrict__ dAP,
    const float *__restrict__ TP, const float *__restrict__ D_chunks, int tc_took, int bh, int slice, int ch_sel,
    int BH) {
    using L = Bwd2Layout<DK>;
    constexpr int NB = DK / 16;
    extern __shared__ float smem[];
    float *sKB = smem + L::oKB, *sQE = smem + L::oQE, *sKI = smem + L::oKI, *sG = smem + L::oG;
    float *sdP = sG, *sdA = sG + kChunk * L::LDC;
    float *sS = smem + L::oS, *sD = smem + L::oD, *sdO = smem + L::odO, *sU = smem + L::oU;
    float *sdR = smem + L::odR, *sA = smem + L::oA, *sP = smem + L::oP;
    float *sEC = smem + L::oVec, *sOne = sEC + DK;
    int *s_flag = reinterpret_cast<int *>(sOne + kChunk);

    const int b = bh / H, h = bh % H;
    const int tid = threadIdx.x, tx = tid & 15, ty = tid >> 4;
    const int vcol0 = slice * kBwd2Dvs;
    const int nchunks = (T + kChunk - 1) / kChunk;
    const size_t BTH = (size_t)BH * T;  // B*H*T token-heads
    const size_t pslice = (size_t)slice * BTH;

    const bool chunk_par = D_chunks != nullptr;
    if (!chunk_par)
        for (int idx = tid; idx < kBwd2Dvs * DK; idx += blockDim.x) {
            const int r = idx / DK, c = idx % DK;
            sD[r * L::LDK + c] = dS_T ? dS_T[((size_t)bh * dv + vcol0 + r) * DK + c] : 0.f;
        }
    if (tid < kChunk) sOne[tid] = 1.f;
    const int ch_first = chunk_par ? ch_sel : nchunks - 1, ch_last = chunk_par ? ch_sel : 0;

#pragma unroll 1
    for (int ch = ch_first; ch >= ch_last; --ch) {
        const int c0 = ch * kChunk;
        const int n = min(kChunk, T - c0);
        const size_t tok0 = ((size_t)b * T + c0) * H + h;
        __syncthreads();
        if (chunk_par) {
            const float *src = D_chunks + (((size_t)bh * nchunks + ch) * dv + vcol0) * DK;
            for (int idx = tid; idx < kBwd2Dvs * DK; idx += blockDim.x)
                sD[(idx / DK) * L::LDK + idx % DK] = src[idx];
        } else if (ch > 0) {  // the previous chunk's inputs -> L2 while this one is reversed
            const size_t tp = tok0 - (size_t)kChunk * H;  // its first token-head
            constexpr int kRowLines = (DK * 4 + 127) / 128, kRowLinesIo = (DK * (int)sizeof(Tio) + 127) / 128;
            for (int idx = tid; idx < kChunk * (2 * kRowLines + 2 * kRowLinesIo + 1); idx += blockDim.x) {
                const int r = idx % kChunk, w = idx / kChunk;
                const size_t row = tp + (size_t)r * H;
                if (w < kRowLines) sm100::prefetch_l2(log_alpha + row * DK + 32 * w);
                else if (w < 2 * kRowLines) sm100::prefetch_l2(bgate + row * DK + 32 * (w - kRowLines));
                else if (w < 2 * kRowLines + kRowLinesIo)
                    sm100::prefetch_l2(k + row * DK + (128 / sizeof(Tio)) * (w - 2 * kRowLines));
                else if (w < 2 * kRowLines + 2 * kRowLinesIo)
                    sm100::prefetch_l2(q + row * DK + (128 / sizeof(Tio)) * (w - 2 * kRowLines - kRowLinesIo));
                else sm100::prefetch_l2(dO + row * dv + vcol0);
            }
            const float *sp = S_chunks + (((size_t)bh * nchunks + ch - 1) * dv + vcol0) * DK;
            for (int l = tid; l < kBwd2Dvs * DK / 32; l += blockDim.x) sm100::prefetch_l2(sp + 32 * l);
        }
        // ---- gates: G (per-channel cumulative log decay), E_C; K, Q, B, dO, S
        if (tid == 0) *s_flag = 0;
#pragma unroll 8
        for (int idx = tid; idx < kChunk * DK; idx += blockDim.x) {
            const int r = idx / DK, j = idx % DK;
            const size_t off = (tok0 + (size_t)r * H) * DK + j;
            const bool ok = r < n;
            sG[r * L::LDK + j] = ok ? log_alpha[off] : 0.f;
            sKB[r * L::LDK + j] = ok ? to_f32(k[off]) * bgate[off] : 0.f;  // K*B, scaled by E below
            sKI[r * L::LDK + j] = ok ? to_f32(k[off]) : 0.f;               // K, divided by E below
            sQE[r * L::LDK + j] = ok ? to_f32(q[off]) : 0.f;               // Q, scaled by E below
        }
        load_tile(sdO, L::LDV, dO + tok0 * dv + vcol0, (size_t)H * dv, n, kBwd2Dvs);
        {
            const float *src = S_chunks + (((size_t)bh * nchunks + ch) * dv + vcol0) * DK;
            for (int idx = tid; idx < kBwd2Dvs * DK; idx += blockDim.x)
                sS[(idx / DK) * L::LDK + idx % DK] = src[idx];
        }
        __syncthreads();
        for (int j = tid; j < DK; j += blockDim.x) {
            float g = 0.f;
            for (int r = 0; r < kChunk; ++r) {
                g += sG[r * L::LDK + j];
                const float e = expf(g);
                sKB[r * L::LDK + j] *= e;
                sQE[r * L::LDK + j] *= e;
                sKI[r * L::LDK + j] = -g <= 80.f ? sKI[r * L::LDK + j] / e : 0.f;
            }
            sEC[j] = expf(g);
            if (-g > 80.f) atomicMax(s_flag, kChunkExact + 1);
            else if (-g > kBwd2TcSpan) atomicMax(s_flag, 1);
        }
        __syncthreads();
        // s_flag: 0 moderate decay, 1 past the tensor-core span, 2 past e^80
        // after the tensor-core gradient kernel, its mode stands (the same
        // thresholds, but the span summed in another order could round across one)
        const int mode = tc_took ? exact_flags[(size_t)bh * nchunks + ch]
                                 : *s_flag == 2 ? kChunkExact : (*s_flag == 1 || !dAP) ? kChunkF32 : kChunkTc;
        if (slice == 0 && tid == 0 && !tc_took) exact_flags[(size_t)bh * nchunks + ch] = mode;
        if (mode == kChunkExact) {  // a channel decays past e^80 inside the chunk: token by token
            gdr2_chunk_reverse_exact<Tio, DK>(n, tok0, H, dv, vcol0, q, k, v, log_alpha, bgate, wgate, dO, smem,
                                              smem + L::odO, sS, sD, dv_out, dw_out, part_qe, part_kb, part_ki,
                                              part_x, pslice);
            continue;
        }

        // ---- P1: A, P (C x C); R = W*V - KBE S^T -> sU.  With TP (tensor-core
        // path, moderate decay) the recompute already formed T = (I + A)^{-1}
        // and P: T goes where A would, and U = T R, dR = T^T dU replace the
        // triangular solves below.
        const bool have_t = TP != nullptr && mode == kChunkTc;
        if (have_t) {
            const float *src = TP + ((size_t)bh * nchunks + ch) * 2 * kChunk * kChunk;
            for (int idx = tid; idx < kChunk * kChunk; idx += blockDim.x) {
                const int r = idx >> 6, i = idx & 63;
                sA[r * L::LDC + i] = src[idx];
                sP[r * L::LDC + i] = src[kChunk * kChunk + idx];
            }
        }
        {
            float aa[4][4] = {}, pp[4][4] = {}, xs[4][2] = {};
#pragma unroll 2
            for (int j = 0; j < (have_t ? 0 : DK); ++j) {
                float kb[4], qe[4], ki[4], sc[2];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    kb[a] = sKB[(ty + 16 * a) * L::LDK + j];
                    qe[a] = sQE[(ty + 16 * a) * L::LDK + j];
                    ki[a] = sKI[(tx + 16 * a) * L::LDK + j];
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) sc[c] = sS[(tx + 16 * c) * L::LDK + j];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        aa[a][c] = fmaf(kb[a], ki[c], aa[a][c]);
                        pp[a][c] = fmaf(qe[a], ki[c], pp[a][c]);
                    }
#pragma unroll
                    for (int c = 0; c < 2; ++c) xs[a][c] = fmaf(kb[a], sc[c], xs[a][c]);
                }
            }
            if (have_t) {  // R alone
#pragma unroll 2
                for (int j = 0; j < DK; ++j) {
                    float kb[4], sc[2];
#pragma unroll
                    for (int a = 0; a < 4; ++a) kb[a] = sKB[(ty + 16 * a) * L::LDK + j];
#pragma unroll
                    for (int c = 0; c < 2; ++c) sc[c] = sS[(tx + 16 * c) * L::LDK + j];
#pragma unroll
                    for (int a = 0; a < 4; ++a)
#pragma unroll
                        for (int c = 0; c < 2; ++c) xs[a][c] = fmaf(kb[a], sc[c], xs[a][c]);
                }
            }
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                if (!have_t) {
#pragma unroll
                    for (int c = 0; c < 4; ++c) {
                        const int i = tx + 16 * c;
                        sA[r * L::LDC + i] = (i < r) ? aa[a][c] : 0.f;
                        sP[r * L::LDC + i] = (i <= r) ? pp[a][c] : 0.f;
                    }
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int cc = tx + 16 * c;
                    float wv = 0.f;
                    if (r < n) {
                        const size_t off = (tok0 + (size_t)r * H) * dv + vcol0 + cc;
                        wv = wgate[off] * to_f32(v[off]);
                    }
                    sU[r * L::LDV + cc] = wv - xs[a][c];
                }
            }
        }
        __syncthreads();

        // ---- P2: U = (I + A)^{-1} R
        if (have_t) {
            float u[4][2] = {};
            for (int i = 0; i < kChunk; ++i) {
                float t[4], rr[2];
#pragma unroll
                for (int a = 0; a < 4; ++a) t[a] = sA[(ty + 16 * a) * L::LDC + i];
#pragma unroll
                for (int c = 0; c < 2; ++c) rr[c] = sU[i * L::LDV + tx + 16 * c];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 2; ++c) u[a][c] = fmaf(t[a], rr[c], u[a][c]);
            }
            __syncthreads();  // every read of R done
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 2; ++c) sU[(ty + 16 * a) * L::LDV + tx + 16 * c] = u[a][c];
            __syncthreads();
        } else {
            fwd_solve<L::LDC, L::LDV, kBwd2Dvs>(sA, sOne, sU);
        }

        // ---- P3: dU = Kt D^T + P^T dO -> sdR ; dP = dO U^T (i <= r) -> sdP
        {
            float du[4][2] = {};
#pragma unroll 2
            for (int j = 0; j < DK; ++j) {
                float kr[4], dd[2];
                const float ec = sEC[j];
#pragma unroll
                for (int a = 0; a < 4; ++a) kr[a] = sKI[(ty + 16 * a) * L::LDK + j] * ec;
#pragma unroll
                for (int c = 0; c < 2; ++c) dd[c] = sD[(tx + 16 * c) * L::LDK + j];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 2; ++c) du[a][c] = fmaf(kr[a], dd[c], du[a][c]);
            }
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
            float dp[4][4] = {};
#pragma unroll 4
            for (int c = 0; c < kBwd2Dvs; ++c) {
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
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = tx + 16 * c;
                    sdP[r * L::LDC + i] = (i <= r) ? dp[a][c] : 0.f;
                }
            }
        }
        __syncthreads();

        // ---- P4: dR = (I + A)^{-T} dU (in sdR)
        if (have_t) {
            float dr[4][2] = {};
            for (int r = 0; r < kChunk; ++r) {
                float t[4], du[2];
#pragma unroll
                for (int a = 0; a < 4; ++a) t[a] = sA[r * L::LDC + ty + 16 * a];
#pragma unroll
                for (int c = 0; c < 2; ++c) du[c] = sdR[r * L::LDV + tx + 16 * c];
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int c = 0; c < 2; ++c) dr[a][c] = fmaf(t[a], du[c], dr[a][c]);
            }
            __syncthreads();  // every read of dU done
#pragma unroll
            for (int a = 0; a < 4; ++a)
#pragma unroll
                for (int c = 0; c < 2; ++c) sdR[(ty + 16 * a) * L::LDV + tx + 16 * c] = dr[a][c];
            __syncthreads();
        } else {
            back_solve<L::LDC, L::LDV, kBwd2Dvs>(sA, sOne, sdR);
        }

        // ---- P5: dA = -dR U^T (i < r) -> sdA ; dV = W*dR, dW = V*dR
        {
            float da[4][4] = {};
#pragma unroll 4
            for (int c = 0; c < kBwd2Dvs; ++c) {
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
#pragma unroll
                for (int c = 0; c < 4; ++c) {
                    const int i = tx + 16 * c;
                    sdA[r * L::LDC + i] = (i < r) ? da[a][c] : 0.f;
                }
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                    const int cc = tx + 16 * c;
                    if (r < n) {
                        const size_t off = (tok0 + (size_t)r * H) * dv + vcol0 + cc;
                        const float dr = sdR[r * L::LDV + cc];
                        dv_out[off] = from_f32<Tio>(wgate[off] * dr);
                        dw_out[off] = to_f32(v[off]) * dr;
                    }
                }
            }
        }
        __syncthreads();

        // ---- P6: slice partials of dKBE, dQE, dKiE (C x DK) and of dE_C (DK).
        // With dAP the products with dA and dP are left to the chunk kernel
        // (bwd2_tc.cuh), which adds the slices' dA and dP first.
        if (mode == kChunkTc) {
            float *dst = dAP + (((size_t)slice * (BTH / T) + bh) * nchunks + ch) * 2 * kChunk * kChunk;
            for (int idx = tid; idx < kChunk * kChunk; idx += blockDim.x) {
                const int r = idx / kChunk, i = idx % kChunk;
                dst[idx] = sdA[r * L::LDC + i];
                dst[kChunk * kChunk + idx] = sdP[r * L::LDC + i];
            }
        }
        {
            float akb[4][NB] = {}, aqe[4][NB] = {}, aki[4][NB] = {}, ud[4][NB] = {};
            // -dR S (-> dKBE), dO S (-> dQE), U D (-> dKiE via Diag(E_C))
#pragma unroll 2
            for (int c = 0; c < kBwd2Dvs; ++c) {
                float dr[4], od[4], ur[4], ss[NB], dd[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = ty + 16 * a;
                    dr[a] = sdR[r * L::LDV + c];
                    od[a] = sdO[r * L::LDV + c];
                    ur[a] = sU[r * L::LDV + c];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    ss[bq] = sS[c * L::LDK + tx + 16 * bq];
                    dd[bq] = sD[c * L::LDK + tx + 16 * bq];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) {
                        akb[a][bq] = fmaf(-dr[a], ss[bq], akb[a][bq]);
                        aqe[a][bq] = fmaf(od[a], ss[bq], aqe[a][bq]);
                        ud[a][bq] = fmaf(ur[a], dd[bq], ud[a][bq]);
                    }
            }
            // dA KiE (-> dKBE), dP KiE (-> dQE), dA^T KBE + dP^T QE (-> dKiE)
#pragma unroll 2
            for (int i = 0; i < (mode == kChunkTc ? 0 : kChunk); ++i) {
                float w_a[4], w_p[4], w_at[4], w_pt[4], ki[NB], kb[NB], qe[NB];
#pragma unroll
                for (int a = 0; a < 4; ++a) {
                    const int r = ty + 16 * a;
                    w_a[a] = sdA[r * L::LDC + i];
                    w_p[a] = sdP[r * L::LDC + i];
                    w_at[a] = sdA[i * L::LDC + r];
                    w_pt[a] = sdP[i * L::LDC + r];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    ki[bq] = sKI[i * L::LDK + tx + 16 * bq];
                    kb[bq] = sKB[i * L::LDK + tx + 16 * bq];
                    qe[bq] = sQE[i * L::LDK + tx + 16 * bq];
                }
#pragma unroll
                for (int a = 0; a < 4; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq) {
                        akb[a][bq] = fmaf(w_a[a], ki[bq], akb[a][bq]);
                        aqe[a][bq] = fmaf(w_p[a], ki[bq], aqe[a][bq]);
                        aki[a][bq] = fmaf(w_at[a], kb[bq], fmaf(w_pt[a], qe[bq], aki[a][bq]));
                    }
            }
            // write the partials; colsum((U D) * KiE) of this thread's rows -> dE_C
            float ecp[NB] = {};
#pragma unroll
            for (int a = 0; a < 4; ++a) {
                const int r = ty + 16 * a;
                const size_t row = pslice * DK + (tok0 + (size_t)r * H) * DK;
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    const int j = tx + 16 * bq;
                    ecp[bq] = fmaf(ud[a][bq], sKI[r * L::LDK + j], ecp[bq]);
                    if (r < n) {
                        part_kb[row + j] = akb[a][bq];
                        part_qe[row + j] = aqe[a][bq];
                        part_ki[row + j] = fmaf(ud[a][bq], sEC[j], aki[a][bq]);
                    }
                }
            }
            // colsum over the 16 row groups (ty) via shared memory, fixed order
            __syncthreads();  // every read of dA / dP done: reuse their space
            float *red = sdP;
#pragma unroll
            for (int bq = 0; bq < NB; ++bq) red[ty * DK + tx + 16 * bq] = ecp[bq];
            __syncthreads();
            for (int j = tid; j < DK; j += blockDim.x) {
                float s = 0.f;
                for (int g = 0; g < 16; ++g) s += red[g * DK + j];
                for (int c = 0; c < kBwd2Dvs; ++c) s = fmaf(sS[c * L::LDK + j], sD[c * L::LDK + j], s);
                part_ec[((size_t)slice * (BTH / T * nchunks) + (size_t)bh * nchunks + ch) * DK + j] = s;
            }
        }
        __syncthreads();

        // ---- P7: D <- D Diag(E_C) + dO^T QE - dR^T KBE (slice rows)
        if (!chunk_par) {
            float dn[2][NB];
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    const int c = ty + 16 * a, j = tx + 16 * bq;
                    dn[a][bq] = sD[c * L::LDK + j] * sEC[j];
                }
#pragma unroll 4
            for (int r = 0; r < kChunk; ++r) {
                float w1[2], w2[2], qr[NB], kr[NB];
#pragma unroll
                for (int a = 0; a < 2; ++a) {
                    w1[a] = sdO[r * L::LDV + ty + 16 * a];
                    w2[a] = -sdR[r * L::LDV + ty + 16 * a];
                }
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) {
                    qr[bq] = sQE[r * L::LDK + tx + 16 * bq];
                    kr[bq] = sKB[r * L::LDK + tx + 16 * bq];
                }
#pragma unroll
                for (int a = 0; a < 2; ++a)
#pragma unroll
                    for (int bq = 0; bq < NB; ++bq)
                        dn[a][bq] = fmaf(w1[a], qr[bq], fmaf(w2[a], kr[bq], dn[a][bq]));
            }
            __syncthreads();  // every read of D done
#pragma unroll
            for (int a = 0; a < 2; ++a)
#pragma unroll
                for (int bq = 0; bq < NB; ++bq) sD[(ty + 16 * a) * L::LDK + tx + 16 * bq] = dn[a][bq];
        }
    }
    __syncthreads();
    if (dS0 && !chunk_par) {
        for (int idx = tid; idx < kBwd2Dvs * DK; idx += blockDim.x) {
            const int r = idx / DK, c = idx % DK;
            dS0[((size_t)bh * dv + vcol0 + r) * DK + c] = sD[r * L::LDK + c];
        }
    }
}

// One CTA per (b*H + h, slice) walking all chunks, or per (b*H + h, slice,
// chunk blockIdx.y) with D_chunks.
template <typename Tio, int DK>
__global__ void __launch_bounds__(kSimtThreads, 1)
gdr2_bwd_simt_kernel(int T, int H, int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                     const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                     const float *__restrict__ bgate, const float *__restrict__ wgate,
                     const Tio *__restrict__ dO, const float *__restrict__ dS_T,
                     const float *__restrict__ S_chunks, Tio *__restrict__ dv_out,
                     float *__restrict__ dw_out, float *__restrict__ dS0, float *__restrict__ part_kb,
                     float *__restrict__ part_qe, float *__restrict__ part_ki, float *__restrict__ part_ec,
                     float *__restrict__ part_x, int *__restrict__ exact_flags, float *__restrict__ dAP,
                     const float *__restrict__ TP, const float *__restrict__ D_chunks) {
    const int nslice = dv / kBwd2Dvs;
    gdr2_bwd_simt_body<Tio, DK>(T, H, dv, q, k, v, log_alpha, bgate, wgate, dO, dS_T, S_chunks, dv_out, dw_out, dS0,
                                part_kb, part_qe, part_ki, part_ec, part_x, exact_flags, dAP, TP, D_chunks, 0,
                                (int)(blockIdx.x / nslice), (int)(blockIdx.x % nslice), (int)blockIdx.y,
                                (int)(gridDim.x / nslice));
}

// The chunks the tensor-core gradient kernel left (todo[0 .. *ntodo), each
// b*H*nchunks + chunk): CTA (slice, g) takes items g, g + gridDim.y, ...
template <typename Tio, int DK>
__global__ void __launch_bounds__(kSimtThreads, 1)
gdr2_bwd_simt_list_kernel(int T, int H, int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                          const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                          const float *__restrict__ bgate, const float *__restrict__ wgate,
                          const Tio *__restrict__ dO, const float *__restrict__ S_chunks,
                          Tio *__restrict__ dv_out, float *__restrict__ dw_out, float *__restrict__ part_kb,
                          float *__restrict__ part_qe, float *__restrict__ part_ki, float *__restrict__ part_ec,
                          float *__restrict__ part_x, int *__restrict__ exact_flags, float *__restrict__ dAP,
                          const float *__restrict__ D_chunks, const int *__restrict__ todo,
                          const int *__restrict__ ntodo, int BH) {
    const int nch = (T + kChunk - 1) / kChunk, n_items = *ntodo;
#pragma unroll 1
    for (int it = blockIdx.y; it < n_items; it += gridDim.y) {
        __syncthreads();  // the previous item is done with shared memory
        const int tile = todo[it];
        gdr2_bwd_simt_body<Tio, DK>(T, H, dv, q, k, v, log_alpha, bgate, wgate, dO, nullptr, S_chunks, dv_out,
                                    dw_out, nullptr, part_kb, part_qe, part_ki, part_ec, part_x, exact_flags, dAP,
                                    nullptr, D_chunks, 1, tile / nch, (int)blockIdx.x, tile % nch, BH);
    }
}

// Sum the per-slice partials in a fixed order and apply the per-element chain
// rule; dlog alpha = the reverse prefix sum of dG per channel inside each
// chunk.  One CTA per (b, h, chunk), one thread per key channel.
template <typename Tio, int DK>
__global__ void __launch_bounds__(DK)
gdr2_bwd_reduce_kernel(int T, int H, int nslice, const Tio *__restrict__ q, const Tio *__restrict__ k,
                       const float *__restrict__ log_alpha, const float *__restrict__ bgate,
                       const float *__restrict__ part_kb, const float *__restrict__ part_qe,
                       const float *__restrict__ part_ki, const float *__restrict__ part_ec,
                       const float *__restrict__ part_x, const int *__restrict__ exact_flags,
                       Tio *__restrict__ dq, Tio *__restrict__ dk, float *__restrict__ dlog_alpha,
                       float *__restrict__ db, size_t BTH) {
    __shared__ float sg[kChunk][DK];
    const int nchunks = (T + kChunk - 1) / kChunk;
    const int ch = blockIdx.x % nchunks;
    const int bh = blockIdx.x / nchunks;
    const int b = bh / H, h = bh % H;
    const int c0 = ch * kChunk, n = min(kChunk, T - c0);
    const size_t tok0 = ((size_t)b * T + c0) * H + h;
    const size_t nbh = BTH / T;
    const int j = threadIdx.x;
    if (exact_flags[(size_t)bh * nchunks + ch] == kChunkExact) {
        // token-by-token partials: S_t^T do (part_qe), X = P^T gk (part_ki),
        // G^T e (part_kb), sum_i P_ij G_ij (part_x)
        for (int r = 0; r < n; ++r) {
            const size_t off = (tok0 + (size_t)r * H) * DK + j;
            float pq = 0.f, x = 0.f, y = 0.f, z = 0.f;
            for (int s = 0; s < nslice; ++s) {
                pq += part_qe[(size_t)s * BTH * DK + off];
                x += part_ki[(size_t)s * BTH * DK + off];
                y += part_kb[(size_t)s * BTH * DK + off];
                z += part_x[(size_t)s * BTH * DK + off];
            }
            const float kv = to_f32(k[off]), bv = bgate[off];
            dq[off] = from_f32<Tio>(pq);
            dk[off] = from_f32<Tio>(fmaf(-bv, x, y));
            db[off] = -kv * x;
            dlog_alpha[off] = fmaf(-bv * kv, x, z);
        }
        return;
    }
    float g = 0.f;
    for (int r = 0; r < n; ++r) {
        g += log_alpha[(tok0 + (size_t)r * H) * DK + j];
        sg[r][j] = g;
    }
    float dec = 0.f;  // dL/dE_C of this channel
    for (int s = 0; s < nslice; ++s) dec += part_ec[(((size_t)s * nbh + bh) * nchunks + ch) * DK + j];
    float suffix = expf(g) * dec;  // dG_C, carried by the chunk's last token
    for (int r = n - 1; r >= 0; --r) {
        const size_t off = (tok0 + (size_t)r * H) * DK + j;
        float skb = 0.f, sqe = 0.f, ski = 0.f;
        for (int s = 0; s < nslice; ++s) {
            skb += part_kb[(size_t)s * BTH * DK + off];
            sqe += part_qe[(size_t)s * BTH * DK + off];
            ski += part_ki[(size_t)s * BTH * DK + off];
        }
        const float G = sg[r][j], e = expf(G), kv = to_f32(k[off]), qv = to_f32(q[off]), bv = bgate[off];
        const float ie = -G <= 80.f ? 1.f / e : 0.f;
        dk[off] = from_f32<Tio>(fmaf(skb * bv, e, ski * ie));
        db[off] = skb * kv * e;
        dq[off] = from_f32<Tio>(sqe * e);
        suffix += skb * kv * bv * e + sqe * qv * e - ski * kv * ie;
        dlog_alpha[off] = suffix;
    }
}

struct Bwd2Workspace {
    float *states, *part_kb, *part_qe, *part_ki, *part_ec, *part_x, *dAP, *TP, *Dch;
    int *flags, *todo, *ntodo;
};

// bf16 with dk = dv = 128 recomputes on the cluster forward and carries dL/dS
// on the tensor cores (bwd2_ds.cuh); the reverse pass then runs per chunk
inline bool bwd2_uses_ds(int dk, int dv, bool bf16) { return bf16 && dk == 128 && dv == 128; }

// bf16 with dk = 128 forms the chunk products on the tensor cores (bwd2_tc.cuh)
inline bool bwd2_uses_tc(int dk, bool bf16) { return bf16 && dk == 128; }

inline size_t bwd2_workspace_bytes(int B, int T, int H, int dk, int dv, bool bf16) {
    const size_t nch = (size_t)(T + kChunk - 1) / kChunk;
    const size_t ns = (size_t)dv / kBwd2Dvs;
    const size_t bth = (size_t)B * T * H;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    return al((size_t)B * H * nch * dv * dk * 4) + 4 * al(ns * bth * dk * 4) + al(ns * B * H * nch * dk * 4) +
           al((2 * (size_t)B * H * nch + 1) * 4) +
           (bwd2_uses_tc(dk, bf16) ? al(ns * B * H * nch * 2 * kChunk * kChunk * 4) +
                                         al((size_t)B * H * nch * 2 * kChunk * kChunk * 4)
                                   : 0) +
           (bwd2_uses_ds(dk, dv, bf16) ? al((size_t)B * H * nch * dv * dk * 4) : 0);
}

inline Bwd2Workspace bwd2_carve(void *ws, int B, int T, int H, int dk, int dv) {
    const size_t nch = (size_t)(T + kChunk - 1) / kChunk;
    const size_t ns = (size_t)dv / kBwd2Dvs;
    const size_t bth = (size_t)B * T * H;
    auto al = [](size_t x) { return (x + 255) / 256 * 256; };
    char *p = static_cast<char *>(ws);
    Bwd2Workspace w;
    w.states = reinterpret_cast<float *>(p);
    p += al((size_t)B * H * nch * dv * dk * 4);
    w.part_kb = reinterpret_cast<float *>(p);
    p += al(ns * bth * dk * 4);
    w.part_qe = reinterpret_cast<float *>(p);
    p += al(ns * bth * dk * 4);
    w.part_ki = reinterpret_cast<float *>(p);
    p += al(ns * bth * dk * 4);
    w.part_ec = reinterpret_cast<float *>(p);
    p += al(ns * B * H * nch * dk * 4);
    w.part_x = reinterpret_cast<float *>(p);
    p += al(ns * bth * dk * 4);
    w.flags = reinterpret_cast<int *>(p);  // then the list of chunks left to the CUDA cores and its length
    w.todo = w.flags + (size_t)B * H * nch;
    w.ntodo = w.todo + (size_t)B * H * nch;
    p += al((2 * (size_t)B * H * nch + 1) * 4);
    w.dAP = reinterpret_cast<float *>(p);  // these two only on the tensor-core path
    p += al(ns * B * H * nch * 2 * kChunk * kChunk * 4);
    w.TP = reinterpret_cast<float *>(p);
    p += al((size_t)B * H * nch * 2 * kChunk * kChunk * 4);
    w.Dch = reinterpret_cast<float *>(p);  // only with the tensor-core dS pass
    return w;
}

template <typename Tio, int DK>
cudaError_t launch_bwd2_simt(int B, int T, int H, int dv, const void *q, const void *k, const void *v,
                             const float *la, const float *bg, const float *wg, const float *S0,
                             const void *dO, const float *dS_T, void *dq, void *dk_out, void *dv_out,
                             float *dla, float *db, float *dw, float *dS0, void *ws, cudaStream_t stream) {
    Bwd2Workspace w = bwd2_carve(ws, B, T, H, DK, dv);
    // 1) forward recompute keeping every chunk's fp32 entry state (the
    //    tensor-core forward for bf16 with dk = dv = 128, else CUDA cores)
    // (the tensor-core forward also leaves every chunk's T and P for step 2)
    const bool tc_fwd = std::is_same<Tio, __nv_bfloat16>::value && DK == 128 && dv == 128;
    cudaError_t err = tc_fwd
                          ? launch_fwd2_tc2(B, T, H, q, k, v, la, bg, wg, S0, nullptr, nullptr, stream, w.states,
                                            w.TP)
                          : launch_gdr2_simt<Tio, DK>(B, T, H, dv, q, k, v, la, bg, wg, S0, nullptr, nullptr, stream,
                                                      w.states);
    if (err != cudaSuccess) return err;
    // 2) with the cluster recompute: every chunk's dL/dS and dS0 by the
    //    tensor-core dS pass, so that step 3 runs per chunk
    if (tc_fwd) {
        err = launch_bwd2_ds(B, T, H, q, k, la, bg, dO, dS_T, dS0, w.Dch, stream);
        if (err != cudaSuccess) return err;
    }
    const bool tc = bwd2_uses_tc(DK, std::is_same<Tio, __nv_bfloat16>::value);
    using L = Bwd2Layout<DK>;
    const int nslice = dv / kBwd2Dvs;
    const int nch = (T + kChunk - 1) / kChunk;
    if (tc_fwd) {
        // 3) every chunk within the tensor-core span: all gradients on the
        //    tensor cores; the others are listed for steps 4 and 5
        err = cudaMemsetAsync(w.ntodo, 0, sizeof(int), stream);
        if (err == cudaSuccess)
            err = launch_bwd2_grad_tc(B, T, H, q, k, v, dO, la, bg, wg, w.states, w.Dch, w.TP, dq, dk_out, dv_out,
                                      dla, db, dw, w.flags, w.todo, w.ntodo, stream);
        if (err != cudaSuccess) return err;
        // 4) the listed chunks: the reverse pass per (slice, chunk) from D_chunks
        //    (a grid of one wave; with nothing listed every CTA exits at once)
        auto lk = gdr2_bwd_simt_list_kernel<Tio, DK>;
        err = cudaFuncSetAttribute(lk, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
        if (err != cudaSuccess) return err;
        const int gy = min(B * H * nch, 148);
        lk<<<dim3((unsigned)nslice, (unsigned)gy), kSimtThreads, L::kBytes, stream>>>(
            T, H, dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k), static_cast<const Tio *>(v), la, bg,
            wg, static_cast<const Tio *>(dO), w.states, static_cast<Tio *>(dv_out), dw, w.part_kb, w.part_qe,
            w.part_ki, w.part_ec, w.part_x, w.flags, w.dAP, w.Dch, w.todo, w.ntodo, B * H);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        err = cudaGetLastError();
        if (err != cudaSuccess) return err;
        // 5) their slices summed, chain rule, dlog alpha
        auto ck = nslice == 4 ? gdr2_bwd_chunk_tc_list_kernel<Tio, 4> : gdr2_bwd_chunk_tc_list_kernel<Tio, 2>;
        err = cudaFuncSetAttribute(ck, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Bwd2TcSmem::kAlloc);
        if (err != cudaSuccess) return err;
        ck<<<(unsigned)min(B * H * nch, 148), kBwd2TcThreads, Bwd2TcSmem::kAlloc, stream>>>(
            T, H, static_cast<const Tio *>(q), static_cast<const Tio *>(k), la, bg, w.part_kb, w.part_qe,
            w.part_ki, w.part_ec, w.part_x, w.flags, w.dAP, static_cast<Tio *>(dq), static_cast<Tio *>(dk_out), dla,
            db, (size_t)B * T * H, w.todo, w.ntodo);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cudaGetLastError();
    }
    // 3) reverse chunk pass per (b, h, slice)
    auto kern = gdr2_bwd_simt_kernel<Tio, DK>;
    err = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)L::kBytes);
    if (err != cudaSuccess) return err;
    kern<<<dim3((unsigned)(B * H * nslice), 1u), kSimtThreads, L::kBytes, stream>>>(
        T, H, dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k), static_cast<const Tio *>(v), la, bg,
        wg, static_cast<const Tio *>(dO), dS_T, w.states, static_cast<Tio *>(dv_out), dw, dS0, w.part_kb,
        w.part_qe, w.part_ki, w.part_ec, w.part_x, w.flags, tc ? w.dAP : nullptr, nullptr, nullptr);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    err = cudaGetLastError();
    if (err != cudaSuccess) return err;
    // 4) sum the slices (and, on the tensor cores, form the products with dA
    //    and dP), chain rule through the gates, dlog alpha by reverse prefix sums
    if (tc) {
        auto ck = nslice == 4 ? gdr2_bwd_chunk_tc_kernel<Tio, 4> : gdr2_bwd_chunk_tc_kernel<Tio, 2>;
        err = cudaFuncSetAttribute(ck, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)Bwd2TcSmem::kAlloc);
        if (err != cudaSuccess) return err;
        ck<<<(unsigned)(B * H * nch), kBwd2TcThreads, Bwd2TcSmem::kAlloc, stream>>>(
            T, H, static_cast<const Tio *>(q), static_cast<const Tio *>(k), la, bg, w.part_kb, w.part_qe,
            w.part_ki, w.part_ec, w.part_x, w.flags, w.dAP, static_cast<Tio *>(dq), static_cast<Tio *>(dk_out), dla,
            db, (size_t)B * T * H);
        g_launches.fetch_add(1, std::memory_order_relaxed);
        return cudaGetLastError();
    }
    gdr2_bwd_reduce_kernel<Tio, DK><<<(unsigned)(B * H * nch), DK, 0, stream>>>(
        T, H, nslice, static_cast<const Tio *>(q), static_cast<const Tio *>(k), la, bg, w.part_kb, w.part_qe,
        w.part_ki, w.part_ec, w.part_x, w.flags, static_cast<Tio *>(dq), static_cast<Tio *>(dk_out), dla, db,
        (size_t)B * T * H);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
