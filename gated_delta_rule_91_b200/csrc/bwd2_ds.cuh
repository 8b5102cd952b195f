// bwd2_ds.cuh -- the Gated DeltaNet-2 backward's dS pass on tcgen05: dL/dS for
// every chunk, carried in TMEM from the last chunk to the first.
//
// The forward's chunk (fwd2_tc2.cuh; Gated Delta Rule-2, "Gated DeltaNet-2:
// Decoupling Erase and Write in Linear Attention",
// agihunt.info/papers/2605.22791) maps S to
//     O = (Q*E) S^T + P U,   S' = S Diag(E_C) + U^T (K*exp(G_C - G)),
//     U = U^g - W S^T,       W = T (K*B*E).
// With D = dL/dS' (the chunk's exit-state gradient), its reverse for S is
//     dU^T = D (K*exp(G_C - G))^T + dO^T P
//     dL/dS = D Diag(E_C) + dO^T (Q*E) - dU^T W,
// which needs only operands bounded at any decay (E, exp(G_C - G) <= 1), so
// every chunk takes it, strongly decaying ones included.
//
// One 2-CTA cluster per (b, h).  The prep CTA is the cluster forward's
// (g2c_prep), walking the chunks from last to first and handing over the
// same slot (K*B*E and Q*E, K*exp(G_C - G), T, P, E_C).  The state CTA keeps
// D in TMEM and, per step:
//   (a) writes D (fp32, the chunk's exit gradient) for the gradient pass,
//       turns it into the bf16 A operand, and scales D by E_C per column;
//   (b) X1 = D (K*exp(G_C - G))^T, X2 = dO^T P, then D += dO^T (Q*E);
//   (d) dU^T = X1 + X2 -> bf16; W (formed one step ahead as W^T =
//       (K*B*E)^T T^T) -> bf16 over the slot's K*B*E;
//   (e) D -= dU^T W.
// The last D is dS0.  Waits are bounded; an abort drains like the forward.
#pragma once
#include <cuda.h>

#include "common.cuh"
#include "fwd2_tc2.cuh"
#include "sm100.cuh"

namespace gdr {

// state TMEM columns (512 allocated): D, X1, X2, W^T
constexpr uint32_t kG2dD = 0, kG2dX1 = 128, kG2dX2 = 192, kG2dW = 256;

// Shared memory follows G2cLayout's state side: slots at S_H, E_C at S_EC, the
// two dO stages at S_V and S_WV, D and then dU^T (bf16) at S_SB.  Barriers
// (S_BAR): dO stage 0, hand_full[2] (where the prep's copies complete), a, b,
// dO stage 1; then the TMEM address and the abort flag.
__device__ __forceinline__ void g2c_dstate(uint8_t *sm, const CUtensorMap *tm_do, int T, int H, int b, int h,
                                           const float *dS_T, float *dS0, float *D_chunks) {
    using L = G2cLayout;
    using namespace sm100;
    constexpr int D = 128;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int wq = warp & 3, wc = warp >> 2;  // TMEM lane quarter, column group (of 4)
    const int row = wq * 32 + lane;           // TMEM lane = value channel c
    const int bh = b * H + h;
    const int nch = (T + kChunk - 1) / kChunk;
    uint64_t *bars = reinterpret_cast<uint64_t *>(sm + L::S_BAR);
    uint64_t *hand_full = bars + 1;  // [2]
    uint64_t *bar_a = bars + 3, *bar_b = bars + 4;
    auto tma_do = [&](int st) { return bars + (st ? 5 : 0); };  // dO stage st
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + 6);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
    const uint32_t sbase = smem_u32(sm);
    auto do_off = [&](int st) { return st ? L::S_WV : L::S_V; };
    auto chunk_of = [&](int n) { return nch - 1 - n; };

    if (tid == 0) {
        for (int i = 0; i < 6; ++i) mbar_init(&bars[i], 1);
        fence_mbar_init();
        *abort_flag = 0;
        prefetch_tmap(tm_do);
        mbar_expect_tx(&hand_full[0], L::H_BYTES);  // arm the slots for steps 0 and 1
        if (nch > 1) mbar_expect_tx(&hand_full[1], L::H_BYTES);
    }
    if (warp == 0) tmem_alloc(tmem_slot, 512);
    tc_before_sync();
    __syncthreads();
    tc_after_sync();
    cluster_sync();
    const uint32_t tmem = *tmem_slot;
    const uint32_t tl = tmem + ((uint32_t)(wq * 32) << 16);
    const uint32_t remote_empty0 = cluster_addr(sm + L::P_BAR + 8 * kG2cBarEmpty, 0);
    const uint32_t remote_landed0 = cluster_addr(sm + L::P_BAR + 8 * kG2cBarLanded, 0);

    {   // seed D = dS_T (or 0)
        float v[32];
        const int col = wc * 32;
        if (dS_T) {
            const float4 *src = reinterpret_cast<const float4 *>(dS_T + ((size_t)bh * D + row) * D + col);
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 x = src[i];
                v[4 * i] = x.x; v[4 * i + 1] = x.y; v[4 * i + 2] = x.z; v[4 * i + 3] = x.w;
            }
        } else {
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] = 0.f;
        }
        tmem_st32(tl + kG2dD + col, v);
        tmem_wait_st();
    }

    int do_issued = 0, do_done = 0;  // dO loads (thread 0)
    auto issue_do = [&](int n) {
        const int st = n & 1;
        mbar_expect_tx(tma_do(st), 16384);
#pragma unroll
        for (int half = 0; half < 2; ++half)
            tma_load_4d(sm + do_off(st) + half * 8192, tm_do, tma_do(st), half * 64, h, chunk_of(n) * kChunk, b);
        ++do_issued;
    };
    // W^T = (K*B*E)^T T^T of step n (thread 0), once its dO tile and slot landed
    auto issue_w = [&](int n) -> bool {
        const int s = n & 1;
        if (!mbar_wait(tma_do(s), (uint32_t)((n >> 1) & 1))) return false;
        ++do_done;
        if (!mbar_wait_cluster(&hand_full[s], (uint32_t)((n >> 1) & 1))) return false;
        if (n + 2 < nch) mbar_arrive_remote(remote_landed0 + 8 * s);  // the prep may restage its slot
        tc_after_sync();
        const uint32_t hs = sbase + L::S_H + s * L::H_TILES;
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
            mma_bf16(tmem + kG2dW, smem_desc_sw128(hs + L::H_KQE + kk * 2048, 16384, 1024),
                     smem_desc_sw128(hs + L::H_TB + kk * 32, 16, 1024), idesc_bf16(128, 64, true, false), kk > 0);
        mma_commit(bar_b);
        return true;
    };

    uint32_t aphase = 0, bphase = 0;
    if (tid == 0) {
        issue_do(0);
        if (nch > 1) issue_do(1);
        if (!issue_w(0)) *abort_flag = 1;
    }
    __syncthreads();

    int n_done = 0;  // steps whose MMAs all completed
#pragma unroll 1
    for (int n = 0; n < nch; ++n) {
        if (*abort_flag) break;
        const int s = n & 1, c = chunk_of(n);
        const uint32_t hs = sbase + L::S_H + s * L::H_TILES;
        const float *ecs = reinterpret_cast<const float *>(sm + L::S_EC + s * L::H_EC);
        const uint32_t dt = sbase + do_off(s);

        // (a) D (the exit-state gradient of chunk c) -> global, -> bf16 operand; D <- D Diag(E_C)
        {
            const int col = wc * 32;
            float v[32];
            tmem_ld32(tl + kG2dD + col, v);
            if (D_chunks) {
                float4 *dst = reinterpret_cast<float4 *>(D_chunks + (((size_t)bh * nch + c) * D + row) * D + col);
#pragma unroll
                for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
            }
            uint8_t *half = sm + L::S_SB + (wc >> 1) * 16384;
#pragma unroll
            for (int q4 = 0; q4 < 4; ++q4) st_bf16x8(half + sw128_offset(row, (wc & 1) * 4 + q4), v + 8 * q4);
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] *= ecs[col + i];
            tmem_st32(tl + kG2dD + col, v);
            tmem_wait_st();
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // (b) X1 = D (K*exp(G_C - G))^T, X2 = dO^T P (-> bar_a); D += dO^T (Q*E)
        if (tid == 0) {
            tc_after_sync();
            const uint32_t sb = sbase + L::S_SB;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
                mma_bf16(tmem + kG2dX1, smem_desc_sw128(sb + (kk >> 2) * 16384 + (kk & 3) * 32, 16, 1024),
                         smem_desc_sw128(hs + L::H_KTL + (kk >> 2) * 8192 + (kk & 3) * 32, 16, 1024),
                         idesc_bf16(128, 64, false, false), kk > 0);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2dX2, smem_desc_sw128(dt + kk * 2048, 8192, 1024),
                         smem_desc_sw128(hs + L::H_PB + kk * 2048, 8192, 1024), idesc_bf16(128, 64, true, true),
                         kk > 0);
            mma_commit(bar_a);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
                mma_bf16(tmem + kG2dD, smem_desc_sw128(dt + kk * 2048, 8192, 1024),
                         smem_desc_sw128(hs + L::H_KQE + 8192 + kk * 2048, 16384, 1024),
                         idesc_bf16(128, 128, true, true), 1);
        }
        __syncwarp();
        // (d) dU^T = X1 + X2 -> bf16 A operand; W of this step over the slot's K*B*E
        if (tid == 0 && (!mbar_wait(bar_a, aphase) || !mbar_wait(bar_b, bphase))) *abort_flag = 1;
        aphase ^= 1;
        bphase ^= 1;
        tc_before_sync();
        __syncthreads();
        if (*abort_flag) break;
        tc_after_sync();
        {
            float x1[16], x2[16];
            tmem_ld16x2(tl + kG2dX1 + wc * 16, x1, tl + kG2dX2 + wc * 16, x2);
#pragma unroll
            for (int i = 0; i < 16; ++i) x1[i] += x2[i];
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(sm + L::S_SB + sw128_offset(row, wc * 2 + ch), x1 + 8 * ch);
            float w[16];
            tmem_ld16(tl + kG2dW + wc * 16, w);
            uint8_t *wdst = sm + L::S_H + s * L::H_TILES + L::H_KQE + (row >> 6) * 16384;
#pragma unroll
            for (int ch = 0; ch < 2; ++ch) st_bf16x8(wdst + sw128_offset(row & 63, wc * 2 + ch), w + 8 * ch);
        }
        fence_async_smem();
        tc_before_sync();
        __syncthreads();

        // (e) D -= dU^T W (W's two 64-row halves of j lie 16 KB apart), then W of the next step
        if (tid == 0) {
            tc_after_sync();
            const uint32_t du = sbase + L::S_SB, w0 = hs + L::H_KQE;
#pragma unroll
            for (int half = 0; half < 2; ++half)
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)
                    mma_bf16(tmem + kG2dD + 64 * half, smem_desc_sw128(du + kk * 32, 16, 1024),
                             smem_desc_sw128(w0 + half * 16384 + kk * 32, 16, 1024),
                             idesc_bf16(128, 64, false, false, true), 1);
            mma_commit(bar_a);
            if (n + 1 < nch && !issue_w(n + 1)) *abort_flag = 1;
        }
        // (g) step n finished: give its slot back, load dO of step n+2 into its stage
        if (tid == 0) {
            if (!*abort_flag && !mbar_wait(bar_a, aphase)) *abort_flag = 1;
            else if (!*abort_flag) {
                n_done = n + 1;
                if (n + 2 < nch) {
                    mbar_expect_tx(&hand_full[s], L::H_BYTES);
                    mbar_arrive_remote(remote_empty0 + 8 * s);
                    issue_do(n + 2);
                }
            }
        }
        aphase ^= 1;
        tc_before_sync();
        __syncthreads();
        tc_after_sync();
    }

    if (!*abort_flag && dS0) {
        float v[32];
        const int col = wc * 32;
        tmem_ld32(tl + kG2dD + col, v);
        float4 *dst = reinterpret_cast<float4 *>(dS0 + ((size_t)bh * D + row) * D + col);
#pragma unroll
        for (int i = 0; i < 8; ++i) dst[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    }
    if (*abort_flag && tid == 0) {
        record_status(GDR_ERR_TIMEOUT);
        // drain: this CTA's dO loads, its MMAs, and the prep CTA's copies into it
        for (int k2 = do_done; k2 < do_issued; ++k2) mbar_wait(tma_do(k2 & 1), (uint32_t)((k2 >> 1) & 1));
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
gdr2_bwd_ds_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_la, const __grid_constant__ CUtensorMap tm_bg,
                   const __grid_constant__ CUtensorMap tm_do, const __nv_bfloat16 *__restrict__ kg,
                   const __nv_bfloat16 *__restrict__ qg, int T, int H, const float *__restrict__ bgate,
                   const float *__restrict__ dS_T, float *__restrict__ dS0, float *__restrict__ D_chunks) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *sm = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                              ~static_cast<uintptr_t>(1023));
    const int bh = blockIdx.x >> 1, b = bh / H, h = bh % H;
    if (sm100::cluster_ctarank() == 0)
        g2c_prep(sm, &tm_q, &tm_k, &tm_la, &tm_bg, T, H, b, h, kg, qg, bgate, nullptr, true);
    else
        g2c_dstate(sm, &tm_do, T, H, b, h, dS_T, dS0, D_chunks);
}

// The dS pass for bf16, dk = dv = 128: D_chunks [B, H, nchunks, 128, 128]
// fp32 receives every chunk's exit-state gradient (nullable), dS0 (nullable)
// the gradient of the entry state.
inline cudaError_t launch_bwd2_ds(int B, int T, int H, const void *q, const void *k, const float *la,
                                  const float *bgate, const void *dO, const float *dS_T, float *dS0,
                                  float *D_chunks, cudaStream_t stream) {
    CUtensorMap mq, mk, mla, mbg, mdo;
    if (!make_token_map(&mq, q, B, T, H, 128) || !make_token_map(&mk, k, B, T, H, 128) ||
        !make_gate_map(&mla, la, B, T, H, 128) || !make_gate_map(&mbg, bgate, B, T, H, 128, 16) ||
        !make_token_map(&mdo, dO, B, T, H, 128))
        return cudaErrorInvalidValue;
    cudaError_t err = cudaFuncSetAttribute(gdr2_bwd_ds_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           (int)G2cLayout::kAlloc);
    if (err != cudaSuccess) return err;
    gdr2_bwd_ds_kernel<<<(unsigned)(2 * B * H), kG2Threads, G2cLayout::kAlloc, stream>>>(
        mq, mk, mla, mbg, mdo, static_cast<const __nv_bfloat16 *>(k), static_cast<const __nv_bfloat16 *>(q), T, H,
        bgate, dS_T, dS0, D_chunks);
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
