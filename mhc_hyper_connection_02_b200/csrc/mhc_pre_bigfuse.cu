// mHC pre-map from an externally computed projection: "FlashInfer mHC module deep dive" §3
// (mhc_pre_big_fuse: dot_mix [num_splits][T][24] and sqrsum [num_splits][T] are given, summed over
// the splits in the kernel, normalised with rstd = 1 / sqrt(sqrsum / k + rms_eps)) and §4
// (mhc_pre_big_fuse_with_prenorm: one dot_mix [T][24], the sum of squares taken from the residual
// inside the kernel, k = 4H). Both then form the gates, the Sinkhorn comb and y = sum_i pre_i R_i
// exactly as mhc_pre does (§3.4 phases, §5.2 reference math).
//
// Kernels (16-byte path: H % 8 == 0, R / y / pre 16-byte aligned):
//   external sqrsum   coef: one token per lane quad sums the splits in order and forms rstd, the
//                     gates and the Sinkhorn comb; then the streaming aggregate of the tensor-core
//                     path (y = bf16_rn(sum_i pre_i R_i), one thread per 8 columns): R read once.
//   with_prenorm      one CTA per token (H <= 8192): each thread loads its columns of all four
//                     streams into registers once, the CTA sums their squares, warp 0 forms rstd
//                     and the pre gates, and y is written from the same registers (R read once);
//                     rstd is parked in post[t][0] for the coef kernel, which then forms post and
//                     the Sinkhorn comb (so no CTA holds its registers through the Sinkhorn).
// Other shapes: one CTA per token looping over the row (sum of squares, then aggregate, which
// finds the row in cache), coefficients included.
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kBfThreads = 256;

// Warp 0: lane quad r = lane & 3 (every quad holds the same token) sums, over the splits in order,
// the components it needs: pre r, post r, comb row r, and (external variant) sqrsum.
struct BfSums {
  float g0, g1, gc[4], ss;
};

__device__ __forceinline__ BfSums bf_sum_splits(const float* __restrict__ dot_mix,
                                                const float* __restrict__ sqrsum, int nsplit,
                                                int64_t T, int64_t t, int r) {
  BfSums a{0.f, 0.f, {0.f, 0.f, 0.f, 0.f}, 0.f};
#pragma unroll 4
  for (int s = 0; s < nsplit; ++s) {
    const float* d = dot_mix + (static_cast<int64_t>(s) * T + t) * kMix;
    a.g0 += __ldg(d + r);
    a.g1 += __ldg(d + 4 + r);
#pragma unroll
    for (int n = 0; n < 4; ++n) a.gc[n] += __ldg(d + 8 + 4 * r + n);
    if (sqrsum) a.ss += __ldg(sqrsum + static_cast<int64_t>(s) * T + t);
  }
  return a;
}

// Post gate and Sinkhorn comb of one token from the quad sums (every lane of warp 0 takes part;
// lanes 0..3 write).
__device__ __forceinline__ void bf_post_comb(const BfSums& a, float rstd, int r,
                                             const float* __restrict__ scale,
                                             const float* __restrict__ base, int64_t t,
                                             const FinishParams& fp, float* __restrict__ post,
                                             float* __restrict__ comb) {
  const int lane = threadIdx.x & 31;
  const float lq = fmaf(a.g1 * rstd, __ldg(scale + 1), __ldg(base + 4 + r));
  const float s2 = __ldg(scale + 2);
  float cr[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) cr[n] = fmaf(a.gc[n] * rstd, s2, __ldg(base + 8 + 4 * r + n));
  sinkhorn_quad(cr, fp.iters, fp.sinkhorn_eps);
  if (lane < 4) {
    post[t * 4 + r] = fp.post_mult * sigmoidf_ieee(lq);
#pragma unroll
    for (int n = 0; n < 4; ++n) comb[t * 16 + r * 4 + n] = cr[n];
  }
}

__device__ __forceinline__ float bf_block_sum(float v, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.f;
#pragma unroll
  for (int w = 0; w < kBfThreads / 32; ++w) s += red[w];  // fixed order
  return s;
}

// Register-resident sum of squares, pre gates and aggregate (with_prenorm): kCh chunks of 8
// columns per thread (H / 8 <= kCh * 256). Writes pre, y and rstd (into post[t][0]).
template <int kCh>
__global__ void __launch_bounds__(kBfThreads, kCh >= 4 ? 2 : 3) pre_prenorm_reg_kernel(
    const float* __restrict__ dot_mix, const uint16_t* __restrict__ R,
    const float* __restrict__ scale, const float* __restrict__ base, uint16_t* __restrict__ y,
    float* __restrict__ pre, float* __restrict__ post, int64_t H8, float rms_eps,
    float pre_eps) {
  __shared__ float red[kBfThreads / 32];
  __shared__ float4 pre_s;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t H = H8 * 8;
  pdl_wait();
  pdl_trigger();

  const uint16_t* Rt = R + t * 4 * H;
  uint4 rv[kCh][4];
#pragma unroll
  for (int c = 0; c < kCh; ++c) {
    const int64_t v = tid + c * kBfThreads;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      rv[c][i] = v < H8 ? ld_stream_ro(Rt + i * H + v * 8) : make_uint4(0u, 0u, 0u, 0u);
  }
  float s0 = 0.f, s1 = 0.f;
#pragma unroll
  for (int c = 0; c < kCh; ++c)
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const uint32_t w4[4] = {rv[c][i].x, rv[c][i].y, rv[c][i].z, rv[c][i].w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float a = bf16_lo(w4[q]), b = bf16_hi(w4[q]);
        s0 = fmaf(a, a, s0);
        s1 = fmaf(b, b, s1);
      }
    }
  const float ss = bf_block_sum(s0 + s1, red);
  if (warp == 0 && lane < 4) {
    const float rstd =
        __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(ss, static_cast<float>(4 * H)) + rms_eps));
    const float pr =
        sigmoidf_ieee(fmaf(__ldg(dot_mix + t * kMix + lane) * rstd, __ldg(scale), __ldg(base + lane))) +
        pre_eps;
    reinterpret_cast<float*>(&pre_s)[lane] = pr;
    pre[t * 4 + lane] = pr;
    if (lane == 0) post[t * 4] = rstd;  // read back by the coef kernel
  }
  __syncthreads();
  const float4 p4 = pre_s;
#pragma unroll
  for (int c = 0; c < kCh; ++c) {
    const int64_t v = tid + c * kBfThreads;
    if (v < H8) {
      const uint32_t* r0 = &rv[c][0].x;
      const uint32_t* r1 = &rv[c][1].x;
      const uint32_t* r2 = &rv[c][2].x;
      const uint32_t* r3 = &rv[c][3].x;
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float lo = p4.x * bf16_lo(r0[q]);
        lo = fmaf(p4.y, bf16_lo(r1[q]), lo);
        lo = fmaf(p4.z, bf16_lo(r2[q]), lo);
        lo = fmaf(p4.w, bf16_lo(r3[q]), lo);
        float hi = p4.x * bf16_hi(r0[q]);
        hi = fmaf(p4.y, bf16_hi(r1[q]), hi);
        hi = fmaf(p4.z, bf16_hi(r2[q]), hi);
        hi = fmaf(p4.w, bf16_hi(r3[q]), hi);
        o[q] = pack_bf16x2(lo, hi);
      }
      st_plain(y + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
    }
  }
}

// Coefficients from split partials, one token per lane quad (8 per warp). kRstdIn: rstd is read
// from post[t][0] (left there by pre_prenorm_reg_kernel) and pre is not written; otherwise rstd
// comes from the summed sqrsum and k, and pre is written too.
template <bool kRstdIn>
__global__ void __launch_bounds__(256) pre_bigfuse_coef_kernel(
    const float* __restrict__ dot_mix, const float* __restrict__ sqrsum, int nsplit, float kden,
    const float* __restrict__ scale, const float* __restrict__ base, float* __restrict__ pre,
    float* __restrict__ post, float* __restrict__ comb, int64_t T, FinishParams fp) {
  const int lane = threadIdx.x & 31;
  const int r = lane & 3;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 2;
  const bool live = t < T;
  const int64_t tt = live ? t : 0;
  pdl_wait();
  pdl_trigger();
  const BfSums a = bf_sum_splits(dot_mix, kRstdIn ? nullptr : sqrsum, nsplit, T, tt, r);
  float rstd;
  if (kRstdIn) {
    rstd = post[tt * 4];
    __syncwarp();  // every lane has read rstd before lane 0 of the quad overwrites it
  } else {
    rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(a.ss, kden) + fp.rms_eps));
  }
  if (!kRstdIn && live)
    pre[t * 4 + r] = sigmoidf_ieee(fmaf(a.g0 * rstd, __ldg(scale), __ldg(base + r))) + fp.pre_eps;
  const float lq = fmaf(a.g1 * rstd, __ldg(scale + 1), __ldg(base + 4 + r));
  const float s2 = __ldg(scale + 2);
  float cr[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) cr[n] = fmaf(a.gc[n] * rstd, s2, __ldg(base + 8 + 4 * r + n));
  sinkhorn_quad(cr, fp.iters, fp.sinkhorn_eps);  // every lane takes part
  if (live) {
    post[t * 4 + r] = fp.post_mult * sigmoidf_ieee(lq);
#pragma unroll
    for (int n = 0; n < 4; ++n) comb[t * 16 + r * 4 + n] = cr[n];
  }
}

// Looping variant for any H and alignment: the sum of squares (when formed here) and the aggregate
// each walk the row; kVec uses 16-byte accesses (H % 8 == 0, R and y 16-byte aligned).
template <bool kVec, bool kPrenorm>
__global__ void __launch_bounds__(kBfThreads) pre_bigfuse_loop_kernel(
    const float* __restrict__ dot_mix, const float* __restrict__ sqrsum, int nsplit, float kden,
    const uint16_t* __restrict__ R, const float* __restrict__ scale,
    const float* __restrict__ base, uint16_t* __restrict__ y, float* __restrict__ pre,
    float* __restrict__ post, float* __restrict__ comb, int64_t T, int64_t H, FinishParams fp) {
  __shared__ float red[kBfThreads / 32];
  __shared__ float4 pre_s;
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  const int warp = tid >> 5, lane = tid & 31, r = lane & 3;
  pdl_wait();
  pdl_trigger();
  const uint16_t* Rt = R + t * 4 * H;

  float ss = 0.f;
  if (kPrenorm) {
    float s0 = 0.f, s1 = 0.f;
    if (kVec) {
      for (int64_t v = tid; v < H / 2; v += kBfThreads) {  // 4H / 8 chunks of the flat row
        const uint4 w = ld_stream_ro(Rt + v * 8);
        const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float a = bf16_lo(w4[q]), b = bf16_hi(w4[q]);
          s0 = fmaf(a, a, s0);
          s1 = fmaf(b, b, s1);
        }
      }
    } else {
      for (int64_t k = tid; k < 4 * H; k += kBfThreads) {
        const float a = bf16_to_f32(Rt[k]);
        s0 = fmaf(a, a, s0);
      }
    }
    ss = bf_block_sum(s0 + s1, red);
  }
  BfSums a{};
  float rstd = 0.f;
  if (warp == 0) {
    a = bf_sum_splits(dot_mix, kPrenorm ? nullptr : sqrsum, nsplit, T, t, r);
    if (!kPrenorm) ss = a.ss;
    rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(ss, kden) + fp.rms_eps));
    const float pr = sigmoidf_ieee(fmaf(a.g0 * rstd, __ldg(scale), __ldg(base + r))) + fp.pre_eps;
    if (lane < 4) {
      reinterpret_cast<float*>(&pre_s)[r] = pr;
      pre[t * 4 + r] = pr;
    }
  }
  __syncthreads();
  const float4 p4 = pre_s;
  if (kVec) {
    for (int64_t v = tid; v < H / 8; v += kBfThreads) {
      uint4 rv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) rv[i] = ld_stream_ro(Rt + i * H + v * 8);
      uint32_t o[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const uint32_t w0 = (&rv[0].x)[q], w1 = (&rv[1].x)[q], w2 = (&rv[2].x)[q],
                       w3 = (&rv[3].x)[q];
        float lo = p4.x * bf16_lo(w0);
        lo = fmaf(p4.y, bf16_lo(w1), lo);
        lo = fmaf(p4.z, bf16_lo(w2), lo);
        lo = fmaf(p4.w, bf16_lo(w3), lo);
        float hi = p4.x * bf16_hi(w0);
        hi = fmaf(p4.y, bf16_hi(w1), hi);
        hi = fmaf(p4.z, bf16_hi(w2), hi);
        hi = fmaf(p4.w, bf16_hi(w3), hi);
        o[q] = pack_bf16x2(lo, hi);
      }
      st_plain(y + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
    }
  } else {
    for (int64_t h = tid; h < H; h += kBfThreads) {
      float acc = p4.x * bf16_to_f32(Rt[h]);
      acc = fmaf(p4.y, bf16_to_f32(Rt[H + h]), acc);
      acc = fmaf(p4.z, bf16_to_f32(Rt[2 * H + h]), acc);
      acc = fmaf(p4.w, bf16_to_f32(Rt[3 * H + h]), acc);
      y[t * H + h] = f32_to_bf16(acc);
    }
  }
  if (warp == 0) bf_post_comb(a, rstd, r, scale, base, t, fp, post, comb);
}

int launch_pre_bigfuse(const BigFuseArgs& a, cudaStream_t s) {
  if (a.T > 0x7fffffff) return -5;
  const FinishParams fp{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};
  const bool pn = a.sqrsum == nullptr;  // with_prenorm
  const bool vec = a.H % 8 == 0 && aligned16(a.R) && aligned16(a.y) && aligned16(a.pre);
  const int64_t H8 = a.H / 8;
  const dim3 tok_grid(static_cast<unsigned>(a.T));
  const dim3 quad_grid(static_cast<unsigned>((4 * a.T + 255) / 256));
  cudaError_t e = cudaSuccess;
  int launches = 0;
  if (vec && !pn) {
    e = launch_pdl(pre_bigfuse_coef_kernel<false>, quad_grid, dim3(256), 0, s, a.dot_mix, a.sqrsum,
                   a.nsplit, a.k, a.hc_scale, a.hc_base, a.pre, a.post, a.comb, a.T, fp);
    const int64_t units = a.T * H8;
    int64_t ab = (units + 255) / 256;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (ab > cap) ab = cap;
    if (e == cudaSuccess)
      e = launch_pdl(pre_agg_vec8_kernel, dim3(static_cast<unsigned>(ab)), dim3(256), 0, s, a.R,
                     static_cast<const float*>(a.pre), a.y, a.T, H8);
    launches = 2;
  } else if (vec && pn && H8 <= 4 * kBfThreads) {
#define MHC_PN_ARGS a.dot_mix, a.R, a.hc_scale, a.hc_base, a.y, a.pre, a.post, H8, a.rms_eps, a.pre_eps
    if (H8 <= kBfThreads)
      e = launch_pdl(pre_prenorm_reg_kernel<1>, tok_grid, dim3(kBfThreads), 0, s, MHC_PN_ARGS);
    else if (H8 <= 2 * kBfThreads)
      e = launch_pdl(pre_prenorm_reg_kernel<2>, tok_grid, dim3(kBfThreads), 0, s, MHC_PN_ARGS);
    else
      e = launch_pdl(pre_prenorm_reg_kernel<4>, tok_grid, dim3(kBfThreads), 0, s, MHC_PN_ARGS);
#undef MHC_PN_ARGS
    if (e == cudaSuccess)
      e = launch_pdl(pre_bigfuse_coef_kernel<true>, quad_grid, dim3(256), 0, s, a.dot_mix,
                     a.sqrsum, 1, a.k, a.hc_scale, a.hc_base, a.pre, a.post, a.comb, a.T, fp);
    launches = 2;
  } else {
#define MHC_BF_ARGS a.dot_mix, a.sqrsum, a.nsplit, a.k, a.R, a.hc_scale, a.hc_base, a.y, a.pre, \
                    a.post, a.comb, a.T, a.H, fp
    if (vec)
      e = pn ? launch_pdl(pre_bigfuse_loop_kernel<true, true>, tok_grid, dim3(kBfThreads), 0, s, MHC_BF_ARGS)
             : launch_pdl(pre_bigfuse_loop_kernel<true, false>, tok_grid, dim3(kBfThreads), 0, s, MHC_BF_ARGS);
    else
      e = pn ? launch_pdl(pre_bigfuse_loop_kernel<false, true>, tok_grid, dim3(kBfThreads), 0, s, MHC_BF_ARGS)
             : launch_pdl(pre_bigfuse_loop_kernel<false, false>, tok_grid, dim3(kBfThreads), 0, s, MHC_BF_ARGS);
#undef MHC_BF_ARGS
    launches = 1;
  }
  if (e != cudaSuccess) return -4;
  note_launches(launches);
  return 0;
}

}  // namespace mhc
