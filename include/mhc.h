/*
 * mhc.h -- C ABI of libmhc.so: the mHC (manifold-constrained hyper-connection) residual mix with
 * HC = 4 streams, on NVIDIA B200 (sm_100a).
 *
 * Two steps make up the path, and a third entry exposes the Sinkhorn step on its own:
 *
 *   mhc_pre       per token: RMS-normalise the flattened [4H] residual row, project it through
 *                 hc_fn [4H,24] to 24 logits, apply hc_scale / hc_base, and emit
 *                 pre = sigmoid(l[0:4]) + pre_eps, post = post_mult * sigmoid(l[4:8]),
 *                 comb = Sinkhorn(exp(l[8:24]) as 4x4) and y = sum_i pre_i * R_i.
 *   mhc_post      out[n][h] = x[h] * post[n] + sum_o R[o][h] * comb[o][n].
 *   mhc_sinkhorn  the Sinkhorn normalisation of caller-given 4x4 logits.
 *
 * Sources (page title and section):
 *   "FlashInfer mHC module deep dive" (www.pwwt.cn/news/5432433):
 *       §1 fixed HC = 4 and the 24-wide mix layout pre(4) | post(4) | comb(16);
 *       §2.1 post-map formula; §2.2 shapes ([T,4] or [T,4,1] post, comb [old][new]);
 *       §2.3 empty input returns without a launch; §3.1-3.2 pre-map parameters and defaults
 *       (rms_eps, sinkhorn eps, sinkhorn_repeat >= 1, eps > 0); §3.4 kernel phases (sum of
 *       squares, rstd, sigmoid gates, softmax with row-max shift, row -> column Sinkhorn rounds,
 *       vec8 aggregate); §4 RMS denominator 4*H; §5.2 test reference math (the Sinkhorn starts
 *       from the row softmax plus eps and divides by plain row and column sums).
 *   rwkv-ops 0.6.1 "rwkv_ops/mhc_kernel/jax_kernel/mhu_jax.py": docstrings of
 *       stream_aggregate (fp32 accumulate, cast back) and mhc_pre_op (H_pre = sigmoid,
 *       H_post = 2 * sigmoid).
 *   "metrale_model_layers/layers/ops/hyper_connection_dispatch.rs": hc_pre_site / hc_post_site
 *       argument lists (device pointers, token count, hidden size, stream; out may alias residual).
 *   "metrale_model_arch/glm5next_mhc.rs": glm_hc_pre (refuse to launch past the scratch
 *       allocation), glm_hc_post (out may alias residual: every stream of an element is read
 *       before it is written), mix_hc.
 *
 * Conventions for every entry point:
 *   - All array pointers are DEVICE pointers into the current CUDA context's memory, dense and
 *     row-major; bf16 arrays are passed as their 16-bit patterns (uint16_t). The caller owns and
 *     allocates every buffer, including the pre-map workspace; the library allocates no device
 *     memory and keeps no state between calls. The one exception is mhc_pre_noalloc, whose fixed
 *     scratch array lives in the library's device image (see its comment).
 *   - Work is enqueued on `stream` (a cudaStream_t; NULL is the legacy default stream) and the call
 *     returns without synchronising. Results are ready when the stream reaches that point.
 *   - Arguments are validated on the host BEFORE anything is launched; on an error nothing is
 *     written and nothing is enqueued. T == 0 returns MHC_OK without a launch.
 *   - The device must be sm_100 (B200); the kernels are built for sm_100a only.
 *   - Return value: MHC_OK (0) or a negative MHC_ERR_* code; mhc_status_string() names it.
 */
#ifndef MHC_H
#define MHC_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MHC_API __attribute__((visibility("default")))
#else
#define MHC_API
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* mhc_stream_t;

enum {
    MHC_HC = 4,   /* streams (fixed) */
    MHC_MIX = 24, /* logits per token: pre(4) | post(4) | comb(16) */
};

enum mhc_status {
    MHC_OK = 0,
    MHC_ERR_INVALID_ARG = -1,         /* null pointer, T < 0, H <= 0, iters < 1, eps <= 0 ... */
    MHC_ERR_WORKSPACE_TOO_SMALL = -2, /* workspace_bytes < mhc_pre_workspace_bytes(T, H) */
    MHC_ERR_ALIAS = -3,               /* an output partially overlaps an input (see each call) */
    MHC_ERR_CUDA = -4,                /* a CUDA runtime call or a launch failed */
    MHC_ERR_UNSUPPORTED = -5,         /* device is not sm_100, or a forced path cannot run */
    MHC_ERR_TIMEOUT = -6,             /* a bounded device-side wait gave up (see mhc_device_status) */
    MHC_ERR_SCRATCH_LIMIT = -7,       /* mhc_pre_noalloc: the size needs more than its fixed scratch */
};

/* Pre-map parameters. Defaults (mhc_default_params): sinkhorn_iters 20 and sinkhorn_eps 1e-6
 * ("FlashInfer mHC module deep dive" §3.2, sinkhorn_repeat / mhc_sinkhorn_eps), rms_eps 1e-6
 * (same table), pre_eps 0 and post_mult 2 (rwkv-ops mhc_pre_op: H_pre = sigmoid,
 * H_post = 2 * sigmoid; FlashInfer's defaults 1e-6 and 1.0 are reachable by setting them). */
typedef struct {
    int sinkhorn_iters; /* >= 1: rounds of (row normalise, column normalise) */
    float sinkhorn_eps; /* > 0: added to every entry of the row softmax before the rounds */
    float rms_eps;      /* > 0: rstd = 1 / sqrt(sum(R^2) / (4H) + rms_eps) */
    float pre_eps;      /* >= 0: added to each pre gate */
    float post_mult;    /* finite: post = post_mult * sigmoid(l[4:8]) */
} mhc_params;

MHC_API mhc_params mhc_default_params(void);

/*
 * mhc_pre -- the fused pre-map (steps: sum of squares -> rstd; projection; logit affine and gates;
 * Sinkhorn; aggregate). "FlashInfer mHC module deep dive" §3.4 and §5.2; rwkv-ops mhc_pre_op.
 *
 *   R        [T][4][H] bf16   residual streams; the row of token t flattened as k = i*H + h
 *   hc_fn    [4H][24]  fp32   projection (row k, logit j)
 *   hc_scale [3]       fp32   logit scales of pre, post, comb, in that order
 *   hc_base  [24]      fp32   logit biases
 *   y        [T][H]    bf16   out: sum_i pre_i * R[t][i][:], fp32 accumulate, rounded to nearest even
 *   pre      [T][4]    fp32   out
 *   post     [T][4]    fp32   out
 *   comb     [T][4][4] fp32   out, [old][new]: comb[o][n] weighs old stream o into new stream n
 *   workspace / workspace_bytes: caller-allocated device scratch of at least
 *            mhc_pre_workspace_bytes(T, H) bytes, 256-byte aligned; its contents on entry do not
 *            matter and on return are unspecified. May be NULL when that size is 0.
 *   p        host pointer to parameters; NULL selects mhc_default_params().
 *
 * Errors: MHC_ERR_INVALID_ARG for a null array, T < 0, H <= 0, or a parameter outside its range;
 * MHC_ERR_WORKSPACE_TOO_SMALL; MHC_ERR_ALIAS when y, pre, post or comb overlaps R or one another.
 * Any H >= 1 is accepted (FlashInfer requires H % 8 == 0; here other H take a scalar path), as is
 * any alignment of the arrays.
 *
 * Kernel choice (MHC_PATH_AUTO): T < 128, odd H or unaligned R / workspace: the CUDA-core split-K
 * path; otherwise the tcgen05 projection, as the single-pass kernel where it is faster (up to
 * about 1.5k tokens with H >= ~2k, 16-byte aligned y, H % 8 == 0), else the split chain. Every
 * path computes the same values within the stated tolerances.
 */
MHC_API int mhc_pre(const uint16_t* R, const float* hc_fn, const float* hc_scale, const float* hc_base,
            uint16_t* y, float* pre, float* post, float* comb, void* workspace,
            size_t workspace_bytes, int64_t T, int64_t H, const mhc_params* p,
            mhc_stream_t stream);

/* Bytes of workspace mhc_pre needs for (T, H): enough for every path mhc_pre or
 * mhc_pre_with_path may take at that size. 0 when T <= 0 or H <= 0. */
MHC_API size_t mhc_pre_workspace_bytes(int64_t T, int64_t H);

/*
 * mhc_post -- the post-map. "FlashInfer mHC module deep dive" §2.1-2.3; glm5next_mhc.rs
 * glm_hc_post; hyper_connection_dispatch.rs hc_post_site.
 *
 *   x     [T][H]     bf16   layer output
 *   R     [T][4][H]  bf16   residual streams
 *   post  [T][4]     fp32   (a [T][4][1] tensor has the same layout)
 *   comb  [T][4][4]  fp32   [old][new]
 *   out   [T][4][H]  bf16   out[t][n][h] = bf16_rn(x*post[n] + sum_o R[o]*comb[o][n]), fp32 math
 *
 * out may be exactly R (in place): each element's four streams are read before it is written.
 * Errors: MHC_ERR_INVALID_ARG (null array, T < 0, H <= 0); MHC_ERR_ALIAS when out overlaps R
 * without being equal to it, or overlaps x, post or comb.
 */
MHC_API int mhc_post(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
             uint16_t* out, int64_t T, int64_t H, mhc_stream_t stream);

/*
 * mhc_sinkhorn -- the Sinkhorn step on its own. "FlashInfer mHC module deep dive" §3.4 (softmax
 * with row-max shift, then row -> column rounds) and §5.2 (its test reference: softmax + eps,
 * then plain row -> column rounds).
 *
 *   logits [T][4][4] fp32   pre-exp logits, [old][new]
 *   comb   [T][4][4] fp32   out: A = softmax(l, each row) + eps; `iters` times { rows /= rowsum;
 *                           columns /= colsum }; may be equal to logits (in place)
 *   H_unused               ignored (kept so every entry takes T and H)
 *
 * Errors: MHC_ERR_INVALID_ARG (null array, T < 0, iters < 1, eps <= 0 or not finite);
 * MHC_ERR_ALIAS when comb overlaps logits without being equal to it.
 */
MHC_API int mhc_sinkhorn(const float* logits, float* comb, int64_t T, int64_t H_unused, int iters,
                 float eps, mhc_stream_t stream);

/* Kernel-path selectors for mhc_pre_with_path / mhc_post_with_path (tests and benchmarks use them
 * to exercise each kernel; mhc_pre / mhc_post are MHC_PATH_AUTO). A forced path that cannot run
 * on the given sizes or alignment returns MHC_ERR_UNSUPPORTED before any launch. */
enum mhc_path {
    MHC_PATH_AUTO = 0,
    /* pre */
    MHC_PRE_PATH_CUDA_CORE = 1, /* fp32 CUDA-core split-K projection + finish kernel */
    MHC_PRE_PATH_TENSOR = 2,    /* tcgen05 projection (exact bf16 x3 split of hc_fn) as the split
                                   chain (MHC_PATH_AUTO may take the single pass instead) */
    MHC_PRE_PATH_TENSOR_SPLIT = 3, /* tcgen05 split-K projection kernel, then a coefficient kernel
                                      and a streaming aggregate kernel; H even */
    MHC_PRE_PATH_TENSOR_FUSED = 4, /* one pass over R: a persistent cooperative kernel (projection
                                      with hc_fn slices resident in shared memory, cross-CTA
                                      reduction, coefficients, aggregate from L2) after a counter
                                      reset; H % 8 == 0, H >= 64, R, y and the workspace 16-byte
                                      aligned; MHC_ERR_UNSUPPORTED, with nothing launched, when
                                      the device cannot hold its grid resident */
    MHC_PRE_PATH_TENSOR_WAVE = 5,  /* one pass over R in wavefront order: every CTA projects a short
                                      K range of the same few token tiles (persistent cooperative
                                      kernel, hc_fn tiles streamed from L2), per-tile counters
                                      release the aggregate units, which re-read the rows from L2;
                                      then the Sinkhorn pass. H % 8 == 0, H >= 64, R, y, comb and
                                      the workspace 16-byte aligned; MHC_ERR_UNSUPPORTED, with
                                      nothing launched, when the device cannot hold its grid
                                      resident */
    /* post */
    MHC_POST_PATH_VEC8 = 11,       /* 16-byte vector loads/stores; H % 8 == 0, 16-byte aligned */
    MHC_POST_PATH_PERSISTENT = 12, /* persistent, bulk-copy (TMA) staged; same requirements */
    MHC_POST_PATH_SCALAR = 13,     /* element-wise; any H and alignment */
};

MHC_API int mhc_pre_with_path(const uint16_t* R, const float* hc_fn, const float* hc_scale,
                      const float* hc_base, uint16_t* y, float* pre, float* post, float* comb,
                      void* workspace, size_t workspace_bytes, int64_t T, int64_t H,
                      const mhc_params* p, int path, mhc_stream_t stream);

MHC_API int mhc_post_with_path(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                       uint16_t* out, int64_t T, int64_t H, int path, mhc_stream_t stream);

/* Reads and clears the device-side status word that bounded waits inside the kernels set when
 * they give up (MHC_OK or MHC_ERR_TIMEOUT). Synchronises `stream` first. Kernels never trap. */
MHC_API int mhc_device_status(mhc_stream_t stream);

/* mhc_selftest_wait_timeout -- health check of the bounded device waits (no counterpart on the
 * pages). Enqueues one kernel whose single thread waits on an mbarrier that nothing arrives at,
 * through the same wait routine every pipeline uses, but with limit_ns (1 us .. 1 s) instead of the
 * library-wide 2 s. The wait runs out, the kernel records MHC_ERR_TIMEOUT in the device status word
 * and returns; no copy is in flight, so the context stays usable. A following mhc_device_status()
 * returns MHC_ERR_TIMEOUT (and clears the word). Errors: MHC_ERR_INVALID_ARG (limit out of range),
 * MHC_ERR_UNSUPPORTED (current device not sm_100), MHC_ERR_CUDA (launch failed). */
MHC_API int mhc_selftest_wait_timeout(int64_t limit_ns, mhc_stream_t stream);

/*
 * mhc_pre_noalloc -- mhc_pre for callers that cannot allocate device memory. No counterpart on the
 * pages: it is an addition of this library.
 *
 * Some callers cannot call cudaMalloc or hand the library a workspace: plugins whose host framework
 * owns every device allocation and whose plugin interface has no workspace argument, and serving
 * loops that must not allocate per call (an allocation can synchronise the device and adds latency
 * to every decode step). This entry computes exactly what mhc_pre computes on its CUDA-core path,
 * but keeps that path's scratch (the split-K partial records, nsplit x T x 128 bytes) in a fixed
 * array of MHC_NOALLOC_SCRATCH_BYTES bytes inside the library's device image instead of a
 * caller workspace. The caller still passes every input and output.
 *
 *   - Sizes whose scratch would exceed MHC_NOALLOC_SCRATCH_BYTES return MHC_ERR_SCRATCH_LIMIT
 *     before anything is launched (every T up to 32768 tokens fits, whatever H; other arguments
 *     and errors are those of mhc_pre). It calls no cudaMalloc, cudaFree or allocating library
 *     routine.
 *   - The array exists on every GPU that loads the library and is held until the process exits.
 *   - Every call looks up the array's device address (cudaGetSymbolAddress, with the device that
 *     owns R current), so a reset device or a recreated context never leaves a stale address
 *     behind. The first lookup on a device can load the library's module there: make the first
 *     call on each device before any stream capture.
 *   - All calls on a device share the one array, which keeps the last call's contents; every record
 *     a call reads is written earlier in the same call, so nothing needs clearing. Calls whose
 *     kernels can overlap on the GPU (different streams without ordering between them) race on the
 *     array and give wrong results; order them on one stream.
 */
#define MHC_NOALLOC_SCRATCH_BYTES (4u << 20)
MHC_API int mhc_pre_noalloc(const uint16_t* R, const float* hc_fn, const float* hc_scale,
                            const float* hc_base, uint16_t* y, float* pre, float* post,
                            float* comb, int64_t T, int64_t H, const mhc_params* p,
                            mhc_stream_t stream);

/*
 * mhc_pre_big_fuse -- the pre-map from a projection computed elsewhere ("FlashInfer mHC module deep
 * dive" §3.1-3.4: mhc_pre_big_fuse; §5.2 reference math). The projection and the sum of squares
 * arrive as num_splits partial sums (for instance from a split-K GEMM), summed here in split order:
 *
 *   dot_mix  [num_splits][T][24] fp32   raw projection partials, sum_k R_flat[t][k] * hc_fn[k][j]
 *   sqrsum   [num_splits][T]     fp32   partials of sum_k R_flat[t][k]^2
 *   num_splits                          1, 2, 4, 8 or 16 (the values the page allows)
 *   k                                   RMS denominator (>= 1; 4H for the mHC row):
 *                                       rstd = 1 / sqrt(sum(sqrsum) / k + rms_eps)
 *   R, hc_scale, hc_base, y, pre, post, comb, p: as mhc_pre (pre is an output here too, although
 *                                       FlashInfer's entry does not return it)
 *
 * logits l = sum(dot_mix) * rstd * hc_scale[group] + hc_base, then gates, Sinkhorn and y as in
 * mhc_pre. Needs no workspace. Any H >= 1 and alignment (H % 8 == 0 with 16-byte aligned R and y
 * takes 16-byte accesses; FlashInfer requires H % 8 == 0).
 * Errors: MHC_ERR_INVALID_ARG (null array, T < 0, H <= 0, num_splits not in {1,2,4,8,16}, k < 1,
 * a parameter outside its range); MHC_ERR_ALIAS when y, pre, post or comb overlaps an input or
 * one another.
 */
MHC_API int mhc_pre_big_fuse(const float* dot_mix, const float* sqrsum, int num_splits, int64_t k,
                             const uint16_t* R, const float* hc_scale, const float* hc_base,
                             uint16_t* y, float* pre, float* post, float* comb, int64_t T,
                             int64_t H, const mhc_params* p, mhc_stream_t stream);

/*
 * mhc_pre_big_fuse_with_prenorm -- as mhc_pre_big_fuse with one split, but the sum of squares is
 * formed here from R and k is 4H ("FlashInfer mHC module deep dive" §4).
 *
 *   dot_mix  [T][24] fp32   raw projection (a [1][T][24] tensor has the same layout)
 */
MHC_API int mhc_pre_big_fuse_with_prenorm(const float* dot_mix, const uint16_t* R,
                                          const float* hc_scale, const float* hc_base,
                                          uint16_t* y, float* pre, float* post, float* comb,
                                          int64_t T, int64_t H, const mhc_params* p,
                                          mhc_stream_t stream);

/*
 * mhc_post_project -- the post-map fused with the next site's projection partials. No entry of
 * this shape is on the pages: pre and post alternate along the layer stack ("FlashInfer mHC
 * module deep dive" §1; glm5next_mhc.rs: the streams glm_hc_post writes are the next residual),
 * and the next pre-map's projection and sum of squares are sums over the new residual row, so
 * they are formed here as split partials while that row is produced; mhc_pre_big_fuse (num_splits
 * = mhc_post_project_splits(T, H), k = 4H) then finishes the next pre-map reading `out` once.
 *
 *   x, R, post, comb, out   as mhc_post; out is bitwise equal to mhc_post's result; out may be R
 *   hc_fn_next  [4H][24] fp32   the next site's projection
 *   dot_mix     [S][T][24] fp32 out: S = mhc_post_project_splits(T, H) (a power of two <= 16)
 *                               partials of sum_k out_flat[t][k] * hc_fn_next[k][j], k = n*H + h,
 *                               over the bf16 values of out; every split is written (zeros where
 *                               a token's row has fewer pieces)
 *   sqrsum      [S][T] fp32     out: partials of sum_k out_flat[t][k]^2
 *   workspace   mhc_post_project_workspace_bytes(T, H) bytes, 256-byte aligned (the split
 *               hc_fn_next operand)
 *
 * Requires H % 8 == 0 and 16-byte aligned x, R, out, post, comb and dot_mix (MHC_ERR_UNSUPPORTED
 * otherwise; use mhc_post then mhc_pre). Errors: MHC_ERR_INVALID_ARG, MHC_ERR_WORKSPACE_TOO_SMALL,
 * MHC_ERR_ALIAS (an output overlapping an input, other than out == R).
 */
MHC_API int mhc_post_project_splits(int64_t T, int64_t H);
MHC_API size_t mhc_post_project_workspace_bytes(int64_t T, int64_t H);
MHC_API int mhc_post_project(const uint16_t* x, const uint16_t* R, const float* post,
                             const float* comb, uint16_t* out, const float* hc_fn_next,
                             float* dot_mix, float* sqrsum, void* workspace,
                             size_t workspace_bytes, int64_t T, int64_t H, mhc_stream_t stream);

/*
 * Backward passes: the exact derivatives of the forward definitions. The pages name backward
 * kernels (rwkv-ops mhu_jax.py: _mhc_post_op_ffi_bwd, mhc_pre_op's VJP) but print no formulas.
 *
 * mhc_post_backward  from d_out [T][4][H] bf16 and the forward's inputs x, R (bf16), post, comb:
 *     d_x[h] = sum_n post[n] d_out[n][h]         (bf16 [T][H], fp32 math, one rounding)
 *     d_R[o][h] = sum_n comb[o][n] d_out[n][h]   (bf16 [T][4][H])
 *     d_post[n] = sum_h x[h] d_out[n][h]         (fp32 [T][4])
 *     d_comb[o][n] = sum_h R[o][h] d_out[n][h]   (fp32 [T][4][4])
 *   Sums over h are fixed-order (deterministic). Errors: MHC_ERR_INVALID_ARG, MHC_ERR_ALIAS (an
 *   output overlapping an input or another output).
 *
 * mhc_pre_backward  from the upstream gradients of the pre-map's outputs -- d_y [T][H] bf16,
 *   d_pre [T][4], d_post [T][4], d_comb [T][4][4] fp32, each optional (NULL = zero) -- and the
 *   forward's inputs R, hc_fn, hc_scale, hc_base with the same params p:
 *     d_R [T][4][H] bf16, d_hc_fn [4H][24] fp32, d_scale [3] fp32, d_base [24] fp32.
 *   The projection is recomputed; gradients flow through the gates (sigmoid), the Sinkhorn rounds
 *   (each normalisation Y = Z / sum has dZ = (dY - sum(dY * Y)) / sum; the starting softmax P
 *   has d_l = P (dA0 - sum_n dA0 P) along the row), the logit
 *   affine, rstd (d_ss = -rstd^3 / (8H) d_rstd) and the aggregate. Token sums are fixed-order.
 *   workspace: mhc_pre_backward_workspace_bytes(T, H) bytes, 256-byte aligned.
 *   Errors: MHC_ERR_INVALID_ARG, MHC_ERR_WORKSPACE_TOO_SMALL, MHC_ERR_ALIAS.
 */
MHC_API int mhc_post_backward(const uint16_t* d_out, const uint16_t* x, const uint16_t* R,
                              const float* post, const float* comb, uint16_t* d_x, uint16_t* d_R,
                              float* d_post, float* d_comb, int64_t T, int64_t H,
                              mhc_stream_t stream);
MHC_API size_t mhc_pre_backward_workspace_bytes(int64_t T, int64_t H);
MHC_API int mhc_pre_backward(const uint16_t* d_y, const float* d_pre, const float* d_post,
                             const float* d_comb, const uint16_t* R, const float* hc_fn,
                             const float* hc_scale, const float* hc_base, uint16_t* d_R,
                             float* d_hc_fn, float* d_scale, float* d_base, void* workspace,
                             size_t workspace_bytes, int64_t T, int64_t H, const mhc_params* p,
                             mhc_stream_t stream);

/*
 * Model-boundary operations: the first layer's expand and the last layer's head. glm5next_mhc.rs
 * glm_hc_expand and hc_head_mean; hyper_connection_dispatch.rs hc_head_site (weighted head).
 * Streams are the library's bf16 [T][4][H] residual (the GLM page keeps them in fp32).
 *
 * mhc_expand     streams[t][i][:] = hidden[t][:] for each of the 4 streams (bitwise copies).
 *                  hidden [T][H] bf16, streams [T][4][H] bf16 out.
 * mhc_head_mean  y[t][:] = bf16_rn(mean_i streams[t][i][:]): the unweighted mean, fp32 sums.
 *                  R [T][4][H] bf16, y [T][H] bf16 out.
 * mhc_head       the weighted collapse: rstd = 1/sqrt(sum(R_flat^2)/(4H) + norm_eps);
 *                  w_i = sigmoid((R_flat . hc_fn[:, i]) * rstd * hc_scale[0] + hc_base[i]) + hc_eps;
 *                  y = bf16_rn(sum_i w_i R_i). The page shows this entry's arguments (hc_fn,
 *                  hc_scale, hc_base, norm eps, hc_eps) but not its kernel; this is the reading in
 *                  which the head is the pre-map's first gate group with its own weights.
 *                  hc_fn [4H][4], hc_scale [1], hc_base [4] fp32; y [T][H] bf16 out; weights
 *                  [T][4] fp32 out, or NULL; workspace of mhc_head_workspace_bytes(T, H) bytes,
 *                  256-byte aligned (contents on entry do not matter).
 * Errors: MHC_ERR_INVALID_ARG (null array, T < 0, H <= 0, norm_eps <= 0, hc_eps < 0, a misaligned
 * workspace); MHC_ERR_WORKSPACE_TOO_SMALL; MHC_ERR_ALIAS when an output overlaps an input.
 */
MHC_API int mhc_expand(const uint16_t* hidden, uint16_t* streams, int64_t T, int64_t H,
                       mhc_stream_t stream);
MHC_API int mhc_head_mean(const uint16_t* R, uint16_t* y, int64_t T, int64_t H,
                          mhc_stream_t stream);
MHC_API size_t mhc_head_workspace_bytes(int64_t T, int64_t H);
MHC_API int mhc_head(const uint16_t* R, const float* hc_fn, const float* hc_scale,
                     const float* hc_base, uint16_t* y, float* weights, void* workspace,
                     size_t workspace_bytes, int64_t T, int64_t H, float norm_eps, float hc_eps,
                     mhc_stream_t stream);

/* Number of kernel launches this process has enqueued through the library so far (all devices,
 * all threads). A diagnostic counter for benchmarks: take the difference around a region. */
MHC_API uint64_t mhc_launch_count(void);

/* Static name of a status code ("MHC_OK", "MHC_ERR_ALIAS", ...). */
MHC_API const char* mhc_status_string(int status);

/* Library version as MAJOR*10000 + MINOR*100 + PATCH. */
MHC_API int mhc_version(void);

#ifdef __cplusplus
}
#endif
#endif /* MHC_H */
