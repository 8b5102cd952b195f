// step_kernel.cuh -- single-token recurrent decode (gdr_step).
//
// One token of the gated delta rule per (b, h) with the fp32 state updated in
// place (Gated DeltaNet review, meaningful96.github.io/nr/GDN, section 3.4;
// recurrent inference keeps only S_t, section 3.1).  Row i of the state
// evolves on its own:
//     a_i = S_i . k,   c_i = S_i . q                (old row, one pass)
//     u_i = beta (v_i - alpha a_i)
//     S_i <- alpha S_i + u_i k
//     o_i = S_i(new) . q = alpha c_i + u_i (k . q)
// so the state is read once and written once, which is the whole cost: the
// step is HBM-bound (2 * dv * dk * 4 bytes of state per head and token).
//
// Mapping: a row of dk fp32 is dk/4 lanes x float4.  A warp keeps kRows rows
// in flight (kLoads float4 loads per lane issued before any use) so that each
// SM has tens of KB of loads outstanding; dots are reduced with warp
// shuffles.  Loads and stores use the streaming cache hints (the state is
// touched once per call).
#pragma once
#include "common.cuh"

namespace gdr {

constexpr int kStepWarps = 4;
constexpr int kStepLoads = 8;  // float4 loads in flight per lane

template <typename Tio, int DK>
struct StepShape {
    static constexpr int kLanesPerRow = DK / 4;               // 32 or 16
    static constexpr int kRowsPerLoad = 32 / kLanesPerRow;    // 1 or 2
    static constexpr int kRowsPerWarp = kStepLoads * kRowsPerLoad;
    static constexpr int kRowsPerCta = kRowsPerWarp * kStepWarps;
};

template <typename Tio, int DK>
__global__ void __launch_bounds__(kStepWarps * 32)
gdr_step_kernel(int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                const float *__restrict__ beta, float *__restrict__ S, Tio *__restrict__ o) {
    using Sh = StepShape<Tio, DK>;
    const int nblk = dv / Sh::kRowsPerCta;
    const int bh = blockIdx.x / nblk;
    const int rblk = blockIdx.x % nblk;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = (lane % Sh::kLanesPerRow) * 4;
    const int sub = lane / Sh::kLanesPerRow;
    const int row0 = rblk * Sh::kRowsPerCta + warp * Sh::kRowsPerWarp;

    const float4 kk = load4(k + (size_t)bh * DK + col);
    const float4 qq = load4(q + (size_t)bh * DK + col);
    const float kq = warp_sum(kk.x * qq.x + kk.y * qq.y + kk.z * qq.z + kk.w * qq.w,
                              Sh::kLanesPerRow);
    const float alpha = expf(log_alpha[bh]);
    const float bt = beta[bh];

    float *Sbh = S + (size_t)bh * dv * DK;
    float4 s[kStepLoads];
#pragma unroll
    for (int l = 0; l < kStepLoads; ++l) {
        const int row = row0 + l * Sh::kRowsPerLoad + sub;
        s[l] = __ldcs(reinterpret_cast<const float4 *>(Sbh + (size_t)row * DK + col));
    }
    float vv[kStepLoads];
#pragma unroll
    for (int l = 0; l < kStepLoads; ++l) {
        const int row = row0 + l * Sh::kRowsPerLoad + sub;
        vv[l] = to_f32(v[(size_t)bh * dv + row]);
    }
#pragma unroll
    for (int l = 0; l < kStepLoads; ++l) {
        const int row = row0 + l * Sh::kRowsPerLoad + sub;
        float a = s[l].x * kk.x + s[l].y * kk.y + s[l].z * kk.z + s[l].w * kk.w;
        float c = s[l].x * qq.x + s[l].y * qq.y + s[l].z * qq.z + s[l].w * qq.w;
        a = warp_sum(a, Sh::kLanesPerRow);
        c = warp_sum(c, Sh::kLanesPerRow);
        const float u = bt * (vv[l] - alpha * a);
        float4 n;
        n.x = fmaf(alpha, s[l].x, u * kk.x);
        n.y = fmaf(alpha, s[l].y, u * kk.y);
        n.z = fmaf(alpha, s[l].z, u * kk.z);
        n.w = fmaf(alpha, s[l].w, u * kk.w);
        __stcs(reinterpret_cast<float4 *>(Sbh + (size_t)row * DK + col), n);
        if ((lane % Sh::kLanesPerRow) == 0)
            o[(size_t)bh * dv + row] = from_f32<Tio>(fmaf(alpha, c, u * kq));
    }
}

template <typename Tio, int DK>
cudaError_t launch_step(int B, int H, int dv, const void *q, const void *k, const void *v,
                        const float *la, const float *beta, float *S, void *o,
                        cudaStream_t stream) {
    using Sh = StepShape<Tio, DK>;
    // consecutive CTAs walk consecutive row blocks of one head (contiguous memory)
    dim3 grid((unsigned)(B * H) * (unsigned)(dv / Sh::kRowsPerCta));
    gdr_step_kernel<Tio, DK><<<grid, kStepWarps * 32, 0, stream>>>(
        dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k), static_cast<const Tio *>(v), la,
        beta, S, static_cast<Tio *>(o));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr

namespace gdr {

// Gated DeltaNet-2 decode (gdr2_step).  One token of the Gated Delta Rule-2
// ("Gated DeltaNet-2: Decoupling Erase and Write in Linear Attention",
// agihunt.info/papers/2605.22791): decay each key channel by alpha, read
// along b*k, write the residual of w*v along k.  Row i of the state:
//     a_i = S_i . (alpha*b*k),   c_i = S_i . (alpha*q)      (old row, one pass)
//     u_i = w_i v_i - a_i
//     S_i <- alpha * S_i + u_i k
//     o_i = S_i(new) . q = c_i + u_i (k . q)
// Same mapping and cost as gdr_step: the fp32 state is read and written once.
template <typename Tio, int DK>
__global__ void __launch_bounds__(kStepWarps * 32)
gdr2_step_kernel(int dv, const Tio *__restrict__ q, const Tio *__restrict__ k,
                 const Tio *__restrict__ v, const float *__restrict__ log_alpha,
                 const float *__restrict__ bgate, const float *__restrict__ wgate, float *__restrict__ S,
                 Tio *__restrict__ o) {
    using Sh = StepShape<Tio, DK>;
    const int nblk = dv / Sh::kRowsPerCta;
    const int bh = blockIdx.x / nblk;
    const int rblk = blockIdx.x % nblk;
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int col = (lane % Sh::kLanesPerRow) * 4;
    const int sub = lane / Sh::kLanesPerRow;
    const int row0 = rblk * Sh::kRowsPerCta + warp * Sh::kRowsPerWarp;

    const float4 kk = load4(k + (size_t)bh * DK + col);
    const float4 qq = load4(q + (size_t)bh * DK + col);
    const float4 la = *reinterpret_cast<const float4 *>(log_alpha + (size_t)bh * DK + col);
    const float4 bb = *reinterpret_cast<const float4 *>(bgate + (size_t)bh * DK + col);
    const float4 al = make_float4(expf(la.x), expf(la.y), expf(la.z), expf(la.w));
    const float4 rk = make_float4(al.x * bb.x * kk.x, al.y * bb.y * kk.y, al.z * bb.z * kk.z, al.w * bb.w * kk.w);
    const float4 rq = make_float4(al.x * qq.x, al.y * qq.y, al.z * qq.z, al.w * qq.w);
    const float kq = warp_sum(kk.x * qq.x + kk.y * qq.y + kk.z * qq.z + kk.w * qq.w, Sh::kLanesPerRow);

    float *Sbh = S + (size_t)bh * dv * DK;
    float4 s[kStepLoads];
#pragma unroll
    for (int l = 0; l < kStepLoads; ++l) {
        const int row = row0 + l * Sh::kRowsPerLoad + sub;
        s[l] = __ldcs(reinterpret_cast<const float4 *>(Sbh + (size_t)row * DK + col));
    }
    float wv[kStepLoads];
#pragma unroll
    for (int l = 0; l < kStepLoads; ++l) {
        const int row = row0 + l * Sh::kRowsPerLoad + sub;
        wv[l] = wgate[(size_t)bh * dv + row] * to_f32(v[(size_t)bh * dv + row]);
    }
#pragma unroll
    for (int l = 0; l < kStepLoads; ++l) {
        const int row = row0 + l * Sh::kRowsPerLoad + sub;
        float a = s[l].x * rk.x + s[l].y * rk.y + s[l].z * rk.z + s[l].w * rk.w;
        float c = s[l].x * rq.x + s[l].y * rq.y + s[l].z * rq.z + s[l].w * rq.w;
        a = warp_sum(a, Sh::kLanesPerRow);
        c = warp_sum(c, Sh::kLanesPerRow);
        const float u = wv[l] - a;
        float4 n;
        n.x = fmaf(al.x, s[l].x, u * kk.x);
        n.y = fmaf(al.y, s[l].y, u * kk.y);
        n.z = fmaf(al.z, s[l].z, u * kk.z);
        n.w = fmaf(al.w, s[l].w, u * kk.w);
        __stcs(reinterpret_cast<float4 *>(Sbh + (size_t)row * DK + col), n);
        if ((lane % Sh::kLanesPerRow) == 0) o[(size_t)bh * dv + row] = from_f32<Tio>(fmaf(u, kq, c));
    }
}

template <typename Tio, int DK>
cudaError_t launch_step2(int B, int H, int dv, const void *q, const void *k, const void *v, const float *la,
                         const float *bgate, const float *wgate, float *S, void *o, cudaStream_t stream) {
    using Sh = StepShape<Tio, DK>;
    dim3 grid((unsigned)(B * H) * (unsigned)(dv / Sh::kRowsPerCta));
    gdr2_step_kernel<Tio, DK><<<grid, kStepWarps * 32, 0, stream>>>(
        dv, static_cast<const Tio *>(q), static_cast<const Tio *>(k), static_cast<const Tio *>(v), la, bgate, wgate,
        S, static_cast<Tio *>(o));
    g_launches.fetch_add(1, std::memory_order_relaxed);
    return cudaGetLastError();
}

}  // namespace gdr
