/*
 * gdr.h -- C ABI of the B200 (sm_100a) gated delta rule library, libgdr.so.
 *
 * The operation (per batch b and head h, state S of dv rows x dk columns):
 *
 *     S_t = S_{t-1} . alpha_t (I - beta_t k_t k_t^T) + beta_t v_t k_t^T,
 *     o_t = S_t q_t                          (readout after the update)
 *
 * with alpha_t = exp(log_alpha_t) in (0,1) and beta_t in (0,1) one scalar per
 * (b, t, h).  Sources: the Gated DeltaNet review at meaningful96.github.io/nr/GDN,
 * section 1 (inputs q, k, v, alpha, beta; outputs S_t and o_t = S_t q_t) and
 * section 3.4 (the gated delta rule); the same rule is stated in section
 * "Method" of "Gated DeltaNet: Merging Gating and the Delta Rule to Beat
 * Mamba2 on Language and Retrieval" (agihunt.info/en/papers/2412.06464).
 * The forward and backward are computed chunkwise (64 tokens per chunk, UT
 * transform / WY form, review section 3.7); the result equals the token
 * recurrence up to rounding.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  * Pointers are DEVICE pointers (cudaMalloc / torch CUDA memory) on the
 *    current device unless stated otherwise.  The caller owns every buffer;
 *    the library never allocates device memory and keeps no state between
 *    calls other than a per-device table of kernel attributes and, once
 *    gdr_seg_fwd has run on a device, one auxiliary stream and two events
 *    there.
 *  * All tensors are dense, row-major, contiguous:
 *      q, k          [B, T, H, dk]      v, o, dO        [B, T, H, dv]
 *      log_alpha     [B, T, H] fp32     beta            [B, T, H] fp32
 *      S0, S_T, dS   [B, H, dv, dk] fp32 (always fp32)
 *    q, k, v, o, dO, dq, dk, dv have the dtype `dt` (GDR_F32 or GDR_BF16).
 *  * q and k are consumed as given: the library does not L2-normalise them
 *    and applies no 1/sqrt(dk) scale (the block normalises them upstream).
 *  * Supported sizes: dk, dv in {64, 128}; B, H >= 1; T >= 1 (a partial last
 *    chunk is handled); B*T*H*max(dk,dv) < 2^31.  Others return
 *    GDR_ERR_UNSUPPORTED (sizes) or GDR_ERR_INVALID_ARGUMENT (non-positive).
 *  * Every pointer must be 16-byte aligned.  Required pointers that are
 *    NULL, or misaligned pointers, return GDR_ERR_INVALID_ARGUMENT.
 *  * Work is enqueued on `stream` (NULL = legacy default stream) and the call
 *    returns without synchronising.  Argument errors are detected on the host
 *    BEFORE anything is launched; nothing is written in that case.
 *  * A launch failure returns GDR_ERR_CUDA.  Kernels that wait on on-chip
 *    barriers give up after a bounded number of polls and record
 *    GDR_ERR_TIMEOUT in a device status word, read by gdr_check_status().
 *  * Outputs must not alias inputs (except S in gdr_step and gdr2_step, o in gdr_seg_fixup
 *    and the conv state in gdr_block_prologue, which are in-out).
 *  * gdr_last_error_string() describes the last non-OK status returned on the
 *    calling thread.
 */
#ifndef GDR_H_
#define GDR_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define GDR_API __attribute__((visibility("default")))
#else
#define GDR_API
#endif

/* Same type as cudaStream_t / CUstream; declared here so the header needs no
 * CUDA include. */
typedef struct CUstream_st *gdr_stream_t;

typedef enum {
    GDR_OK = 0,
    GDR_ERR_INVALID_ARGUMENT = 1, /* NULL/misaligned pointer, non-positive size */
    GDR_ERR_UNSUPPORTED = 2,      /* size or dtype this build does not handle  */
    GDR_ERR_WORKSPACE = 3,        /* workspace NULL or smaller than required  */
    GDR_ERR_CUDA = 4,             /* a CUDA runtime call or launch failed      */
    GDR_ERR_TIMEOUT = 5           /* a bounded on-chip wait gave up (device)   */
} gdr_status;

typedef enum { GDR_F32 = 0, GDR_BF16 = 1 } gdr_dtype;

/*
 * Chunkwise forward.
 *   in : q, k [B,T,H,dk]; v [B,T,H,dv] (dtype dt); log_alpha, beta [B,T,H]
 *        fp32; S0 [B,H,dv,dk] fp32 or NULL (zero initial state).
 *   out: o [B,T,H,dv] (dtype dt); S_T [B,H,dv,dk] fp32, or NULL to skip.
 *   workspace: optional device scratch.  gdr_fwd_workspace_bytes(...) is
 *        nonzero only for a long sequence over few heads (bf16, dk = dv =
 *        128, T/R >= 2048 tokens and 4*B*H*R <= the SM count for some R >= 2;
 *        GDR_FWD_SPLIT=off in the environment turns it off).  Given at
 *        least that many bytes, the call runs R segments of the sequence in
 *        parallel (the sequence split below, inside one GPU: both passes on
 *        two streams, the scan of the segment maps and the correction);
 *        with less, or NULL, it runs the sequence as one chain.  The
 *        results agree up to rounding.
 */
GDR_API gdr_status gdr_fwd(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                   const void *q, const void *k, const void *v,
                   const float *log_alpha, const float *beta, const float *S0,
                   void *o, float *S_T, void *workspace, size_t workspace_bytes,
                   gdr_stream_t stream);
GDR_API size_t gdr_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt);

/*
 * Single-token recurrent decode (recurrent inference, review section 3.1:
 * keeping only S_t makes token-by-token inference possible).
 *   in : q, k [B,H,dk]; v [B,H,dv] (dtype dt); log_alpha, beta [B,H] fp32.
 *   in/out: S [B,H,dv,dk] fp32, advanced by one token in place.
 *   out: o [B,H,dv] (dtype dt) = S_t q.
 */
GDR_API gdr_status gdr_step(int B, int H, int dk, int dv, gdr_dtype dt,
                    const void *q, const void *k, const void *v,
                    const float *log_alpha, const float *beta,
                    float *S, void *o, gdr_stream_t stream);

/*
 * Backward of gdr_fwd (reverse mode; the pages give none, it is the chain
 * rule of the recurrence).  Loss gradients are taken with respect to the
 * given q, k, v, log_alpha, beta and S0.
 *   in : the forward's inputs (S0 may be NULL = 0); dO [B,T,H,dv] (dtype dt);
 *        dS_T [B,H,dv,dk] fp32 or NULL (zero).
 *   out: dq, dk [B,T,H,dk], dv [B,T,H,dv] (dtype dt); dlog_alpha, dbeta
 *        [B,T,H] fp32; dS0 [B,H,dv,dk] fp32 or NULL to skip.
 *   workspace: at least gdr_bwd_workspace_bytes(...) bytes (required): it
 *        holds every chunk's starting state and per-slice partial gradients.
 */
GDR_API gdr_status gdr_bwd(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                   const void *q, const void *k, const void *v,
                   const float *log_alpha, const float *beta, const float *S0,
                   const void *dO, const float *dS_T,
                   void *dq, void *dk_out, void *dv_out,
                   float *dlog_alpha, float *dbeta, float *dS0,
                   void *workspace, size_t workspace_bytes, gdr_stream_t stream);
GDR_API size_t gdr_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt);

/*
 * gdr_bwd without caller-provided workspace.  This entry point has no
 * counterpart in the pages; it exists for callers that cannot allocate
 * device memory at the point where they need the backward -- for example
 * code running inside a pool or arena that owns all device memory, an
 * embedding runtime that forbids cudaMalloc after start-up, or an
 * allocation-free hot loop.  The caller still owns and passes every input
 * and output buffer (same arguments and meaning as gdr_bwd, minus the
 * workspace).
 *
 * The scratch it needs (chunk-entry states and per-slice partial
 * gradients) lives in a fixed 64 MiB static device array inside libgdr.so,
 * so every GPU that loads the library holds those 64 MiB until the
 * process exits.  Problems whose scratch exceeds 64 MiB
 * (gdr_bwd_workspace_bytes(...) > 64 MiB) are rejected on the host with
 * GDR_ERR_WORKSPACE before anything is launched.  It calls no cudaMalloc,
 * cudaFree or other allocating routine.
 *
 * The first call on each device resolves the array's device address
 * (cudaGetSymbolAddress) with that device current; make that first call
 * before any stream capture.  The library keeps that address for the rest
 * of the process: after cudaDeviceReset on a device the module is loaded
 * again and the array may move, so do not call this entry point on a device
 * that has been reset.  All calls share the one array and it keeps
 * the last call's contents (nothing in it needs to start at zero: every
 * byte a call reads is written earlier in the same call), so calls whose
 * work overlaps on the GPU (different streams, or threads racing on one
 * device) race on the scratch: serialise them.
 */
GDR_API gdr_status gdr_bwd_noalloc(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                   const void *q, const void *k, const void *v,
                   const float *log_alpha, const float *beta, const float *S0,
                   const void *dO, const float *dS_T,
                   void *dq, void *dk_out, void *dv_out,
                   float *dlog_alpha, float *dbeta, float *dS0, gdr_stream_t stream);

/*
 * Gated Delta Rule-2 forward ("Gated DeltaNet-2: Decoupling Erase and Write
 * in Linear Attention", agihunt.info/papers/2605.22791, Gated Delta Rule-2
 * paragraph): per token, decay each key channel, read along b_t*k_t, write the
 * residual of w_t*v_t along k_t:
 *     S' = S_{t-1} Diag(alpha_t);  S_t = S' - (S'(b_t*k_t) - w_t*v_t) k_t^T;
 *     o_t = S_t q_t.
 *   in : q, k, v as gdr_fwd; log_alpha [B,T,H,dk] fp32 (per key channel);
 *        b [B,T,H,dk] fp32 (erase gate); w [B,T,H,dv] fp32 (write gate);
 *        S0 [B,H,dv,dk] fp32 or NULL.
 *   out: o [B,T,H,dv] (dtype dt); S_T fp32 or NULL.
 */
GDR_API gdr_status gdr2_fwd(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                    const void *q, const void *k, const void *v,
                    const float *log_alpha, const float *b, const float *w,
                    const float *S0, void *o, float *S_T,
                    void *workspace, size_t workspace_bytes, gdr_stream_t stream);
GDR_API size_t gdr2_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt);

/*
 * Gated Delta Rule-2 backward: gradients of gdr2_fwd (the pages give no
 * backward; this is the chain rule of the step above).
 *   in : the inputs of gdr2_fwd; dO [B,T,H,dv] (dtype dt); dS_T [B,H,dv,dk]
 *        fp32 or NULL (= 0).
 *   out: dq, dk_out [B,T,H,dk] and dv_out [B,T,H,dv] (dtype dt);
 *        dlog_alpha, db [B,T,H,dk] fp32; dw [B,T,H,dv] fp32;
 *        dS0 [B,H,dv,dk] fp32 or NULL.
 * The caller-owned workspace (at least gdr2_bwd_workspace_bytes) holds the
 * recomputed forward's chunk-entry states and per-slice partial sums.  Any
 * decay is handled: a 64-token chunk in which some key channel decays by more
 * than e^80 (where the chunk form's per-channel factors would overflow) is
 * differentiated token by token instead.
 */
GDR_API gdr_status gdr2_bwd(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                    const void *q, const void *k, const void *v,
                    const float *log_alpha, const float *b, const float *w, const float *S0,
                    const void *dO, const float *dS_T,
                    void *dq, void *dk_out, void *dv_out,
                    float *dlog_alpha, float *db, float *dw, float *dS0,
                    void *workspace, size_t workspace_bytes, gdr_stream_t stream);
GDR_API size_t gdr2_bwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt);

/*
 * Gated DeltaNet-2 single-token decode, state updated in place:
 *     S' = S Diag(alpha),  S <- S' - (S'(b*k) - w*v) k^T,  o = S q
 * (the Gated Delta Rule-2 paragraph of "Gated DeltaNet-2: Decoupling Erase
 * and Write in Linear Attention", agihunt.info/papers/2605.22791; the same
 * step gdr2_fwd takes per token).
 *   in : q, k [B,H,dk]; v [B,H,dv] (dtype dt); log_alpha, b [B,H,dk] fp32
 *        (per key channel); w [B,H,dv] fp32 (per value channel).
 *   in/out: S [B,H,dv,dk] fp32.   out: o [B,H,dv] (dtype dt).
 *   Errors: the common size rules (T = 1).
 */
GDR_API gdr_status gdr2_step(int B, int H, int dk, int dv, gdr_dtype dt,
                     const void *q, const void *k, const void *v,
                     const float *log_alpha, const float *b, const float *w,
                     float *S, void *o, gdr_stream_t stream);

/*
 * Block prologue: the q/k/v paths of a Gated DeltaNet block between the input
 * projections and the recurrence, one pass over HBM.
 *     q = L2(SiLU(ShortConv(xq))),  k = L2(SiLU(ShortConv(xk))),
 *     v = SiLU(ShortConv(xv))
 * Source: the Gated DeltaNet review (meaningful96.github.io/nr/GDN), section
 * 3.8 "Gated DeltaNet Block", and the block-design paragraph of "Gated
 * DeltaNet-2: Decoupling Erase and Write in Linear Attention"
 * (agihunt.info/papers/2605.22791).  The pages fix no widths or epsilons:
 *   * ShortConv is a depthwise causal convolution along time of width K
 *     (1..8), in a framework Conv1d's cross-correlation convention:
 *         z[t, c] = bias[c] + sum_{j<K} w[c, j] * x[t-K+1+j, c],
 *     tokens before the first coming from the carried conv state;
 *   * SiLU(z) = z / (1 + exp(-z));
 *   * L2(y) = y / sqrt(sum y^2 + eps) over each head's d channels, per token.
 *   in : xq, xk [B,T,H,dk]; xv [B,T,H,dv] (dtype dt): the projected inputs.
 *        wq, wk [H*dk, K]; wv [H*dv, K] fp32 conv taps (row = channel h*d+i).
 *        bq, bk [H*dk]; bv [H*dv] fp32 conv biases; each may be NULL (zero).
 *        conv_state_in [B, K-1, H*(2*dk+dv)] (dtype dt; channels ordered q,
 *        k, v): the K-1 inputs before token 0, oldest first; NULL = zeros.
 *        eps >= 0 (0 is the plain definition; an all-zero head then gives NaN).
 *   out: q, k [B,T,H,dk]; v [B,T,H,dv] (dtype dt).
 *        conv_state_out (layout of conv_state_in, may be NULL): the last K-1
 *        inputs of the concatenation (conv_state_in, x), for the next segment
 *        or decode token.  It MAY equal conv_state_in (in-place update).
 *   Both states are ignored when K = 1.  Other outputs must not alias inputs.
 *   Errors: K outside 1..8 or the common size rules -> GDR_ERR_UNSUPPORTED;
 *   negative or non-finite eps -> GDR_ERR_INVALID_ARGUMENT.
 */
GDR_API gdr_status gdr_block_prologue(int B, int T, int H, int dk, int dv, int K, gdr_dtype dt,
                              const void *xq, const void *xk, const void *xv,
                              const float *wq, const float *wk, const float *wv,
                              const float *bq, const float *bk, const float *bv,
                              const void *conv_state_in, void *conv_state_out, float eps,
                              void *q, void *k, void *v, gdr_stream_t stream);

/*
 * Backward of gdr_block_prologue (same page sections).  For each stream, with
 * z = ShortConv(x), u = SiLU(z), n = sqrt(sum_head u^2 + eps), y = u / n
 * (q, k) or y = u (v), and the incoming gradient dy of y:
 *     du = (dy - y (y . dy)) / n   (q, k; per token and head)   du = dy (v)
 *     dz = du sig(z) (1 + z (1 - sig(z))),  sig = 1/(1 + e^-z)
 *     dx[s, c] = sum_j w[c, j] dz[s+K-1-j, c] over output tokens in [0, T)
 *     dw[c, j] = sum_{b,t} dz[t, c] x[t-K+1+j, c]      dbias[c] = sum_{b,t} dz[t, c]
 * where x at tokens -(K-1)..-1 is conv_state_in.  dconv_state_out, if given,
 * is the gradient of the returned state: it adds to dx of the last K-1
 * inputs (or to dconv_state_in where those were carried in, T < K-1).
 *   in : the forward's inputs (xq, xk, xv, taps, biases, conv_state_in, eps);
 *        dyq, dyk [B,T,H,dk]; dyv [B,T,H,dv] (dtype dt);
 *        dconv_state_out [B, K-1, H*(2*dk+dv)] (dtype dt) or NULL (zero).
 *   out: dxq, dxk [B,T,H,dk]; dxv [B,T,H,dv] (dtype dt);
 *        dwq, dwk [H*dk, K]; dwv [H*dv, K] fp32, overwritten;
 *        dbq, dbk, dbv fp32 or NULL (not written);
 *        dconv_state_in [B, K-1, H*(2*dk+dv)] (dtype dt) or NULL (not written).
 *   workspace: device scratch of gdr_block_prologue_bwd_workspace_bytes(H,
 *        dk, dv, K) bytes: per-block partial sums of dw and dbias, which a
 *        second launch adds in a fixed order (repeated calls give identical
 *        bits).  No output may alias an input or another output.
 *   Errors: as gdr_block_prologue; workspace NULL or short -> GDR_ERR_WORKSPACE.
 */
GDR_API gdr_status gdr_block_prologue_bwd(int B, int T, int H, int dk, int dv, int K, gdr_dtype dt,
                                  const void *xq, const void *xk, const void *xv,
                                  const float *wq, const float *wk, const float *wv,
                                  const float *bq, const float *bk, const float *bv,
                                  const void *conv_state_in, float eps,
                                  const void *dyq, const void *dyk, const void *dyv,
                                  const void *dconv_state_out,
                                  void *dxq, void *dxk, void *dxv,
                                  float *dwq, float *dwk, float *dwv,
                                  float *dbq, float *dbk, float *dbv,
                                  void *dconv_state_in, void *workspace, size_t workspace_bytes,
                                  gdr_stream_t stream);
/* 0 for unsupported sizes. */
GDR_API size_t gdr_block_prologue_bwd_workspace_bytes(int H, int dk, int dv, int K);

/*
 * Block epilogue: the recurrent output's normalisation and output gate, one
 * pass over HBM (same sources as gdr_block_prologue):
 *     y = o / sqrt(mean_i o_i^2 + eps) * weight * SiLU(g)
 * per (token, head) over the dv channels.  The output projection that follows
 * is a plain matrix product and not part of this library.
 *   in : o [B,T,H,dv] (dtype dt, the output of gdr_fwd / gdr2_fwd);
 *        g [B,T,H,dv] (dtype dt) the output-gate projection, or NULL for a
 *        plain RMSNorm; weight [dv] fp32, shared by all heads; eps >= 0.
 *   out: y [B,T,H,dv] (dtype dt); must not alias o or g.
 *   Errors: dv not 64 or 128 and the common size rules -> GDR_ERR_UNSUPPORTED;
 *   negative or non-finite eps -> GDR_ERR_INVALID_ARGUMENT.
 */
GDR_API gdr_status gdr_block_epilogue(int B, int T, int H, int dv, gdr_dtype dt, const void *o,
                              const void *g, const float *weight, float eps, void *y,
                              gdr_stream_t stream);

/*
 * Backward of gdr_block_epilogue (the same normalised, gated output of the
 * Gated DeltaNet block: the Gated DeltaNet review, meaningful96.github.io/nr/GDN,
 * section 3.8).  With a = o r, r = 1/sqrt(mean_i o_i^2 + eps), s = SiLU(g)
 * (s = 1 without a gate), sig = 1/(1 + e^-g) and an incoming dy:
 *     dg      = dy a weight sig (1 + g (1 - sig))
 *     do      = r (dy weight s - a mean_i(dy_i weight_i s_i a_i))
 *     dweight = sum over all B*T*H rows of dy a s.
 *   in:  o, g (or NULL), dy [B,T,H,dv] dtype dt; weight [dv] fp32; eps >= 0
 *        as in the forward.
 *   out: dO [B,T,H,dv] dtype dt; dg likewise (NULL exactly when g is NULL);
 *        dweight [dv] fp32, overwritten (not accumulated).
 *   workspace: device scratch of gdr_block_epilogue_bwd_workspace_bytes(dv)
 *        bytes (per-block partial sums of dweight, which a second launch adds
 *        in a fixed order, so repeated calls give identical bits).
 *   Errors: as gdr_block_epilogue; g and dg not both given or both NULL ->
 *   GDR_ERR_INVALID_ARGUMENT; workspace NULL or short -> GDR_ERR_WORKSPACE.
 */
GDR_API gdr_status gdr_block_epilogue_bwd(int B, int T, int H, int dv, gdr_dtype dt, const void *o,
                                  const void *g, const float *weight, float eps, const void *dy,
                                  void *dO, void *dg, float *dweight, void *workspace,
                                  size_t workspace_bytes, gdr_stream_t stream);
/* 0 for an unsupported dv. */
GDR_API size_t gdr_block_epilogue_bwd_workspace_bytes(int dv);

/*
 * Sequence split: one sequence divided into R consecutive segments, one per
 * process/GPU, each run by its owner, with one exchange of small matrices.
 * For one (b, h) the rule over a segment maps the incoming state affinely,
 *     S_out = S_in M + N,
 * N (dv x dk) being the segment's final state from S_in = 0 and M (dk x dk)
 * the product of the per-token factors alpha_t (I - beta_t k_t k_t^T) in
 * token order; in the chunkwise form of the Gated DeltaNet review
 * (meaningful96.github.io/nr/GDN, section 3.7) it is the product of the
 * chunks' (gamma_C I - W^T K) factors.  The readout is affine too:
 *     o_t = o_t(S_in = 0) + S_in q~_t,   q~_t = M_<=t q_t,
 * and the rule run with v = 0 from S_in = I (dv = dk) returns q~ as its
 * outputs and M as its final state.  Per rank r of R:
 *   1. gdr_seg_fwd on the segment -> o(0), q~, N, M;
 *   2. all-gather (M, N) of every segment in order (the caller's collective);
 *   3. gdr_seg_combine(R, r, ...) -> S_in of segment r (and the final state);
 *   4. gdr_seg_fixup -> o = o(0) + S_in q~.
 * The result equals gdr_fwd over the whole sequence up to rounding.
 */

/* Both forward passes of one segment (tokens of this segment only, T of
 * them, inputs laid out as for gdr_fwd; S_in is not an input).
 *   out: o0 [B,T,H,dv] (dtype dt) outputs from S_in = 0;
 *        qt [B,T,H,dk] (dtype dt) q~_t = M_<=t q_t;
 *        N [B,H,dv,dk] fp32; M [B,H,dk,dk] fp32.
 * workspace (>= gdr_seg_fwd_workspace_bytes) holds a zero value tensor and the
 * identity state of the second pass.  The two passes are independent: the
 * second runs on the library's auxiliary stream of the device, forked from and
 * joined back into `stream` with events, so both small grids share the GPU
 * and `stream` sees the call complete as usual.  Errors as for gdr_fwd, plus
 * GDR_ERR_WORKSPACE. */
GDR_API gdr_status gdr_seg_fwd(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                       const void *q, const void *k, const void *v,
                       const float *log_alpha, const float *beta,
                       void *o0, void *qt, float *N, float *M,
                       void *workspace, size_t workspace_bytes, gdr_stream_t stream);
GDR_API size_t gdr_seg_fwd_workspace_bytes(int B, int T, int H, int dk, int dv, gdr_dtype dt);

/* The sequential combine of the segment maps, fp32: S = S0 (NULL: zeros);
 * for j = 0 .. R-1: S = S M_j + N_j.
 *   in : M [R,B,H,dk,dk], N [R,B,H,dv,dk] (segment j's gdr_seg_fwd outputs at
 *        index j); S0 [B,H,dv,dk] or NULL; 0 <= r < R.
 *   out: S_in [B,H,dv,dk] = S before segment r (may be NULL);
 *        S_T [B,H,dv,dk] = S after segment R-1, the state after the whole
 *        sequence (may be NULL; not both).
 *   Errors: r outside 0..R-1 or both outputs NULL -> GDR_ERR_INVALID_ARGUMENT;
 *   sizes as for gdr_fwd. */
GDR_API gdr_status gdr_seg_combine(int R, int r, int B, int H, int dk, int dv,
                           const float *M, const float *N, const float *S0,
                           float *S_in, float *S_T, gdr_stream_t stream);

/* The correction of one segment's outputs: o[b,t,h,:] += S_in[b,h] qt[b,t,h,:]
 * in fp32, rounded once to dtype dt.
 *   in : qt [B,T,H,dk] (gdr_seg_fwd's q~), S_in [B,H,dv,dk] fp32.
 *   in/out: o [B,T,H,dv] (gdr_seg_fwd's o0 on entry).  Sizes as gdr_fwd. */
GDR_API gdr_status gdr_seg_fixup(int B, int T, int H, int dk, int dv, gdr_dtype dt,
                         const void *qt, const float *S_in, void *o, gdr_stream_t stream);

/* Synchronise `stream`, then read and clear the device status word that
 * kernels set when a bounded wait gives up (GDR_ERR_TIMEOUT).  Returns
 * GDR_OK, that status, or GDR_ERR_CUDA if the synchronisation itself failed. */
GDR_API gdr_status gdr_check_status(gdr_stream_t stream);

/* Test hook for the timeout path: launches a one-thread kernel that waits on
 * an on-chip barrier nothing ever arrives on, with a bound of `timeout_ms`
 * milliseconds (1..10000).  The wait runs out, the kernel records
 * GDR_ERR_TIMEOUT in the device status word and returns normally: no fault,
 * no trap, the context stays usable.  A following gdr_check_status(stream)
 * returns GDR_ERR_TIMEOUT (and clears the word). */
GDR_API gdr_status gdr_debug_wait_timeout(int timeout_ms, gdr_stream_t stream);

/* Text for the last non-OK status returned on this host thread. */
GDR_API const char *gdr_last_error_string(void);

/* Number of kernels this library has launched in this process (all
 * threads); lets a caller count launches inside a timed region. */
GDR_API uint64_t gdr_launch_count(void);

/* Library version, (major << 16) | minor. */
GDR_API int gdr_version(void);

#ifdef __cplusplus
}
#endif
#endif /* GDR_H_ */
