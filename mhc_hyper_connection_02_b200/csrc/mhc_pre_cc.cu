// mHC pre-map on CUDA cores (fp32): split-K projection partials, then a finish kernel.
//
// This is the path for decode-sized token counts, where the bytes are dominated by hc_fn (read
// once, in fp32, spread over every SM), and the GPU cross-check for the tensor-core path (the
// glm5next_mhc.rs pattern of checking a fused kernel against a split pair, hc_mix + hc_finish).
//
//   partial kernel  grid (ceil(T/32), nsplit), 8 warps. Lane = token, warp = slice of this split's
//                   K range. Each lane accumulates, in fp32 and in k order, the sum of squares and
//                   the 24 dot products of its token's row with hc_fn (hc_fn rows are read with
//                   warp-uniform 16-byte loads, i.e. broadcast). The 8 warps' partials are summed
//                   in warp order through shared memory; record [split][t][32] = raw[0..23], ss.
//   finish kernel   grid (T, 1 + ceil(H/2048)). Every block sums the split records of its token in
//                   a fixed order (so every block computes bit-identical coefficients), forms
//                   rstd = 1/sqrt(ss/(4H) + rms_eps) and the logits l_j = raw_j*rstd*scale[g(j)] +
//                   base[j]. Block 0 writes pre, post and comb (Sinkhorn in one lane quad); blocks
//                   1.. aggregate y = sum_i pre_i*R_i over a 2048-column slice.
//
// "FlashInfer mHC module deep dive" §3.3-3.4 (split reduction of dot_mix / sqrsum, rstd, gates,
// Sinkhorn, vec8 aggregate), §4 (RMS denominator 4H); glm5next_mhc.rs glm_hc_pre (mix, finish).
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kCcWarps = 8;
constexpr int kCcTokens = 32;
constexpr int kCcRec = 32;            // floats per (split, token) record: raw[24], ss, padding
constexpr int64_t kCcPlanCtas = 148;  // target CTAs for the split plan (device independent)
constexpr int kCcLoadBatch = 19;      // records a finish warp loads before adding (148 / 8 rounded up)
constexpr int kAggCols = 2048;        // columns per aggregate block (256 threads x 8)

struct CcPlan {
  int64_t nsplit;
  int64_t KS;
};

static CcPlan cc_plan(int64_t T, int64_t H) {
  const int64_t K = 4 * H;
  const int64_t groups = (T + kCcTokens - 1) / kCcTokens;
  const int64_t kblocks = (K + 63) / 64;
  int64_t nsplit = (kCcPlanCtas + groups - 1) / groups;
  if (nsplit < 1) nsplit = 1;
  if (nsplit > kblocks) nsplit = kblocks;
  int64_t KS = (K + nsplit - 1) / nsplit;
  KS = (KS + 63) / 64 * 64;
  nsplit = (K + KS - 1) / KS;
  return {nsplit, KS};
}

size_t pre_cc_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0) return 0;
  const CcPlan p = cc_plan(T, H);
  return static_cast<size_t>(p.nsplit) * static_cast<size_t>(T) * kCcRec * sizeof(float);
}

template <bool kAlignedW>
__device__ __forceinline__ void cc_accumulate(float r, const float* w, float (&acc)[kMix],
                                              float& ss) {
  ss = fmaf(r, r, ss);
  if (kAlignedW) {
#pragma unroll
    for (int q = 0; q < 6; ++q) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(w) + q);
      acc[4 * q + 0] = fmaf(r, v.x, acc[4 * q + 0]);
      acc[4 * q + 1] = fmaf(r, v.y, acc[4 * q + 1]);
      acc[4 * q + 2] = fmaf(r, v.z, acc[4 * q + 2]);
      acc[4 * q + 3] = fmaf(r, v.w, acc[4 * q + 3]);
    }
  } else {
#pragma unroll
    for (int j = 0; j < kMix; ++j) acc[j] = fmaf(r, __ldg(w + j), acc[j]);
  }
}

template <bool kVecR, bool kAlignedW>
__global__ void __launch_bounds__(256) pre_cc_partial_kernel(const uint16_t* __restrict__ R,
                                                             const float* __restrict__ W,
                                                             float* __restrict__ part, int64_t T,
                                                             int64_t K, int64_t KS) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  __shared__ float red[kCcWarps][kCcTokens][25];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kCcTokens;
  const int64_t s = blockIdx.y;
  const int64_t t = t0 + lane;
  const int64_t kb = s * KS;
  const int64_t ke = min(K, kb + KS);
  const int64_t KW = KS / kCcWarps;  // multiple of 8
  const int64_t k0 = kb + warp * KW;
  const int64_t k1 = min(ke, k0 + KW);

  float acc[kMix];
#pragma unroll
  for (int j = 0; j < kMix; ++j) acc[j] = 0.f;
  float ss = 0.f;
  if (t < T) {
    const uint16_t* row = R + t * K;
    int64_t k = k0;
    if (kVecR) {
      for (; k + 8 <= k1; k += 8) {
        const uint4 v = ld_stream_ro(row + k);
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          cc_accumulate<kAlignedW>(bf16_lo(u[e]), W + (k + 2 * e) * kMix, acc, ss);
          cc_accumulate<kAlignedW>(bf16_hi(u[e]), W + (k + 2 * e + 1) * kMix, acc, ss);
        }
      }
    }
    for (; k < k1; ++k) cc_accumulate<kAlignedW>(bf16_to_f32(row[k]), W + k * kMix, acc, ss);
  }
#pragma unroll
  for (int j = 0; j < kMix; ++j) red[warp][lane][j] = acc[j];
  red[warp][lane][24] = ss;
  __syncthreads();
  for (int idx = threadIdx.x; idx < kCcTokens * 25; idx += blockDim.x) {
    const int tl = idx / 25;
    const int j = idx - tl * 25;
    if (t0 + tl >= T) continue;
    float v = 0.f;
#pragma unroll
    for (int w = 0; w < kCcWarps; ++w) v += red[w][tl][j];
    part[(s * T + t0 + tl) * kCcRec + j] = v;
  }
}

// Decode-sized calls (T <= 8): lanes run along K instead of along tokens. Thread i of split s
// owns k = s*KS + i (and k + 256 when KS > 256): it loads that k's 24 hc_fn weights once and the
// row's value of every token up front, then per token forms its 24 products and its square, and a
// butterfly reduce-scatter over the warp (31 shuffles) leaves lane j holding the warp's sum of
// component j. The 8 warp sums are added in warp order. One hc_fn read per call, every load
// issued before any is used: the step is a few round trips of latency.
constexpr int kKlPer = 2;          // k values per thread at most (KS <= 512)
constexpr int kKlMaxTokens = 8;    // above this the staged lane-per-token kernel is faster (measured)

template <bool kAlignedW>
__global__ void __launch_bounds__(256) pre_cc_partial_klane_kernel(const uint16_t* __restrict__ R,
                                                                   const float* __restrict__ W,
                                                                   float* __restrict__ part,
                                                                   int64_t T, int64_t K,
                                                                   int64_t KS) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  __shared__ float red[kCcWarps][kCcTokens][kCcRec + 1];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t s = blockIdx.y;
  const int64_t kb = s * KS;
  const int64_t ke = min(K, kb + KS);
  float w[kKlPer][kMix];
  float rv[kKlPer][kCcTokens];
#pragma unroll
  for (int i = 0; i < kKlPer; ++i) {
    const int64_t k = kb + threadIdx.x + i * 256;
    const bool ok = k < ke;
    if (kAlignedW) {
#pragma unroll
      for (int q = 0; q < 6; ++q) {
        const float4 v = ok ? __ldg(reinterpret_cast<const float4*>(W + k * kMix) + q)
                            : make_float4(0.f, 0.f, 0.f, 0.f);
        w[i][4 * q] = v.x, w[i][4 * q + 1] = v.y, w[i][4 * q + 2] = v.z, w[i][4 * q + 3] = v.w;
      }
    } else {
#pragma unroll
      for (int j = 0; j < kMix; ++j) w[i][j] = ok ? __ldg(W + k * kMix + j) : 0.f;
    }
#pragma unroll
    for (int t = 0; t < kCcTokens; ++t)
      rv[i][t] = (ok && t < T) ? bf16_to_f32(R[t * K + k]) : 0.f;
  }
#pragma unroll
  for (int t = 0; t < kCcTokens; ++t) {
    if (t >= T) break;
    float v[32];
#pragma unroll
    for (int j = 0; j < kMix; ++j) v[j] = rv[0][t] * w[0][j];
    v[kMix] = rv[0][t] * rv[0][t];
#pragma unroll
    for (int i = 1; i < kKlPer; ++i) {
#pragma unroll
      for (int j = 0; j < kMix; ++j) v[j] = fmaf(rv[i][t], w[i][j], v[j]);
      v[kMix] = fmaf(rv[i][t], rv[i][t], v[kMix]);
    }
#pragma unroll
    for (int j = kMix + 1; j < 32; ++j) v[j] = 0.f;
    // Reduce-scatter: after the step over offset o, a lane keeps the half of its list that its
    // lane bit o selects; after five steps lane j holds component j summed over the warp.
#pragma unroll
    for (int o = 16; o >= 1; o >>= 1) {
      const bool upper = (lane & o) != 0;
#pragma unroll
      for (int i = 0; i < o; ++i) {
        const float keep = upper ? v[o + i] : v[i];
        const float give = upper ? v[i] : v[o + i];
        v[i] = keep + __shfl_xor_sync(0xffffffffu, give, o);
      }
    }
    red[warp][t][lane] = v[0];
  }
  __syncthreads();
  for (int idx = threadIdx.x; idx < T * 25; idx += blockDim.x) {
    const int tl = idx / 25;
    const int j = idx - tl * 25;
    float acc = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kCcWarps; ++w8) acc += red[w8][tl][j];
    part[(s * T + tl) * kCcRec + j] = acc;
  }
}

// Decode-sized calls with more tokens (8 < T <= 32): lane = token as in pre_cc_partial_kernel,
// but the split's hc_fn rows (KS x 24 fp32, at most 48 KB) are first copied into shared memory
// with coalesced loads, so the loop reads them from shared memory (one broadcast per row) instead
// of waiting on global memory for every eight k.
constexpr int kStMaxKS = 512;

template <bool kVecR, bool kAlignedW>
__global__ void __launch_bounds__(256) pre_cc_partial_staged_kernel(const uint16_t* __restrict__ R,
                                                                    const float* __restrict__ W,
                                                                    float* __restrict__ part,
                                                                    int64_t T, int64_t K,
                                                                    int64_t KS) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  __shared__ __align__(16) float sm[kStMaxKS * kMix];  // W slice, then the warp partial sums
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t s = blockIdx.y;
  const int64_t kb = s * KS;
  const int64_t ke = min(K, kb + KS);
  const int nw = static_cast<int>((ke - kb) * kMix);
  const int64_t KW = KS / kCcWarps;  // multiple of 8
  const int64_t k0 = kb + warp * KW;
  const int64_t k1 = min(ke, k0 + KW);
  const int64_t t = lane;
  // The lane's row values are loaded before the W slice is staged, so both round trips overlap.
  constexpr int kStVec = kStMaxKS / kCcWarps / 8;  // 16-byte chunks per lane at most
  uint4 rq[kStVec];
#pragma unroll
  for (int q = 0; q < kStVec; ++q)
    rq[q] = (kVecR && t < T && k0 + 8 * q + 8 <= k1) ? ld_stream_ro(R + t * K + k0 + 8 * q)
                                                      : make_uint4(0u, 0u, 0u, 0u);
  if (kAlignedW) {
    const float4* src = reinterpret_cast<const float4*>(W + kb * kMix);
    for (int i = threadIdx.x; i < nw / 4; i += blockDim.x)
      reinterpret_cast<float4*>(sm)[i] = __ldg(src + i);
  } else {
    for (int i = threadIdx.x; i < nw; i += blockDim.x) sm[i] = __ldg(W + kb * kMix + i);
  }
  __syncthreads();
  float acc[kMix];
#pragma unroll
  for (int j = 0; j < kMix; ++j) acc[j] = 0.f;
  float ss = 0.f;
  auto add_row = [&](float r, int64_t k) {
    const float4* w4 = reinterpret_cast<const float4*>(sm + (k - kb) * kMix);
    ss = fmaf(r, r, ss);
#pragma unroll
    for (int q = 0; q < 6; ++q) {
      const float4 v = w4[q];
      acc[4 * q + 0] = fmaf(r, v.x, acc[4 * q + 0]);
      acc[4 * q + 1] = fmaf(r, v.y, acc[4 * q + 1]);
      acc[4 * q + 2] = fmaf(r, v.z, acc[4 * q + 2]);
      acc[4 * q + 3] = fmaf(r, v.w, acc[4 * q + 3]);
    }
  };
  if (t < T) {
    const uint16_t* row = R + t * K;
    int64_t k = k0;
    if (kVecR) {
#pragma unroll
      for (int q = 0; q < kStVec; ++q) {
        if (k + 8 > k1) break;
        const uint32_t u[4] = {rq[q].x, rq[q].y, rq[q].z, rq[q].w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          add_row(bf16_lo(u[e]), k + 2 * e);
          add_row(bf16_hi(u[e]), k + 2 * e + 1);
        }
        k += 8;
      }
    }
    for (; k < k1; ++k) add_row(bf16_to_f32(row[k]), k);
  }
  __syncthreads();  // every warp is done with the W slice
  float (*red)[kCcTokens][25] = reinterpret_cast<float (*)[kCcTokens][25]>(sm);
#pragma unroll
  for (int j = 0; j < kMix; ++j) red[warp][lane][j] = acc[j];
  red[warp][lane][24] = ss;
  __syncthreads();
  for (int idx = threadIdx.x; idx < T * 25; idx += blockDim.x) {
    const int tl = idx / 25;
    const int j = idx - tl * 25;
    float v = 0.f;
#pragma unroll
    for (int w8 = 0; w8 < kCcWarps; ++w8) v += red[w8][tl][j];
    part[(s * T + tl) * kCcRec + j] = v;
  }
}

struct FinishParams {
  int iters;
  float sinkhorn_eps;
  float rms_eps;
  float pre_eps;
  float post_mult;
};

// Per-token coefficient step shared by the finish kernels: from the summed record (raw[24] in lanes
// 0..23, ss in lane 24) compute the logits; block 0 (write_all) stores pre/post/comb. Returns the
// four pre gates in shared memory. Must be called by one whole warp.
__device__ __forceinline__ void finish_coefficients(float tot, int64_t t, int64_t K,
                                                    const float* __restrict__ scale,
                                                    const float* __restrict__ base,
                                                    const FinishParams& fp, bool write_all,
                                                    float* __restrict__ pre,
                                                    float* __restrict__ post,
                                                    float* __restrict__ comb, float* pre_smem) {
  const int lane = threadIdx.x & 31;
  const float ss = __shfl_sync(0xffffffffu, tot, 24);
  const float rstd = __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(ss, static_cast<float>(K)) + fp.rms_eps));
  float l = 0.f;
  if (lane < kMix) {
    const int g = lane < 4 ? 0 : (lane < 8 ? 1 : 2);
    l = fmaf(tot * rstd, __ldg(scale + g), __ldg(base + lane));
  }
  const float sg = sigmoidf_ieee(l);
  if (lane < 4) pre_smem[lane] = sg + fp.pre_eps;
  if (write_all) {
    if (lane < 4) pre[t * 4 + lane] = sg + fp.pre_eps;
    else if (lane < 8) post[t * 4 + (lane - 4)] = fp.post_mult * sg;
    float a[4];
    const int o = lane & 3;
#pragma unroll
    for (int n = 0; n < 4; ++n) a[n] = __shfl_sync(0xffffffffu, l, 8 + 4 * o + n);
    sinkhorn_quad(a, fp.iters, fp.sinkhorn_eps);
    if (lane < 4) {
      float* dst = comb + t * 16 + lane * 4;
#pragma unroll
      for (int n = 0; n < 4; ++n) dst[n] = a[n];
    }
  }
}

// Eight columns of y = bf16_rn(sum_i pre_i R_i) from the four streams' 16-byte chunks.
__device__ __forceinline__ uint4 agg8(const uint4 (&r)[4], const float (&p)[4]) {
  uint32_t o[4];
  const uint32_t* r0 = &r[0].x;
  const uint32_t* r1 = &r[1].x;
  const uint32_t* r2 = &r[2].x;
  const uint32_t* r3 = &r[3].x;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    float lo = p[0] * bf16_lo(r0[e]);
    lo = fmaf(p[1], bf16_lo(r1[e]), lo);
    lo = fmaf(p[2], bf16_lo(r2[e]), lo);
    lo = fmaf(p[3], bf16_lo(r3[e]), lo);
    float hi = p[0] * bf16_hi(r0[e]);
    hi = fmaf(p[1], bf16_hi(r1[e]), hi);
    hi = fmaf(p[2], bf16_hi(r2[e]), hi);
    hi = fmaf(p[3], bf16_hi(r3[e]), hi);
    o[e] = pack_bf16x2(lo, hi);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

// y[t][h0..h0+8) = bf16_rn(sum_i pre_i * R[t][i][..]) for the columns this thread owns.
template <bool kVec>
__device__ __forceinline__ void aggregate_cols(const uint16_t* __restrict__ R,
                                               uint16_t* __restrict__ y, int64_t t, int64_t H,
                                               int64_t c0, int64_t c1, const float (&p)[4]) {
  const uint16_t* rr = R + t * 4 * H;
  uint16_t* yy = y + t * H;
  if (kVec) {
    for (int64_t h = c0 + threadIdx.x * 8; h + 8 <= c1; h += blockDim.x * 8) {
      uint4 r[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) r[i] = ld_stream_ro(rr + i * H + h);
      st_plain(yy + h, agg8(r, p));
    }
  } else {
    for (int64_t h = c0 + threadIdx.x; h < c1; h += blockDim.x) {
      float acc = p[0] * bf16_to_f32(rr[h]);
      acc = fmaf(p[1], bf16_to_f32(rr[H + h]), acc);
      acc = fmaf(p[2], bf16_to_f32(rr[2 * H + h]), acc);
      acc = fmaf(p[3], bf16_to_f32(rr[3 * H + h]), acc);
      yy[h] = f32_to_bf16(acc);
    }
  }
}

template <bool kVec>
__global__ void __launch_bounds__(256) pre_cc_finish_kernel(
    const uint16_t* __restrict__ R, const float* __restrict__ part, int64_t nsplit,
    const float* __restrict__ scale, const float* __restrict__ base, uint16_t* __restrict__ y,
    float* __restrict__ pre, float* __restrict__ post, float* __restrict__ comb, int64_t T,
    int64_t H, FinishParams fp) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  __shared__ float red[kCcWarps][25];
  __shared__ float pre_s[4];
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t t = blockIdx.x;
  float v = 0.f;
  if (lane < 25) {
    // Warp w adds the records of splits w, w + 8, w + 16, ... in that order. A batch of up to
    // kCcLoadBatch of them is loaded before any is added, so one batch (all of them for the split
    // counts the plan produces) costs one round trip to L2.
    for (int64_t s0 = warp; s0 < nsplit; s0 += static_cast<int64_t>(kCcWarps) * kCcLoadBatch) {
      float r[kCcLoadBatch];
#pragma unroll
      for (int i = 0; i < kCcLoadBatch; ++i) {
        const int64_t s = s0 + static_cast<int64_t>(i) * kCcWarps;
        r[i] = s < nsplit ? part[(s * T + t) * kCcRec + lane] : 0.f;
      }
#pragma unroll
      for (int i = 0; i < kCcLoadBatch; ++i) v += r[i];
    }
  }
  if (lane < 25) red[warp][lane] = v;
  __syncthreads();
  if (warp == 0) {
    float tot = 0.f;
    if (lane < 25) {
#pragma unroll
      for (int w = 0; w < kCcWarps; ++w) tot += red[w][lane];
    }
    finish_coefficients(tot, t, 4 * H, scale, base, fp, blockIdx.y == 0, pre, post, comb, pre_s);
  }
  __syncthreads();
  if (blockIdx.y == 0) return;
  const float p[4] = {pre_s[0], pre_s[1], pre_s[2], pre_s[3]};
  const int64_t c0 = static_cast<int64_t>(blockIdx.y - 1) * kAggCols;
  const int64_t c1 = min(H, c0 + kAggCols);
  aggregate_cols<kVec>(R, y, t, H, c0, c1, p);
}

// Split-K projection partials: records [nsplit][T][32] (raw[24], ss) at the workspace start.
int launch_cc_projection(const PreArgs& a, cudaStream_t s, float** part_out, int* nrec_out) {
  const CcPlan plan = cc_plan(a.T, a.H);
  const int64_t K = 4 * a.H;
  float* part = static_cast<float*>(a.workspace);
  const int64_t groups = (a.T + kCcTokens - 1) / kCcTokens;
  if (groups > 0x7fffffff || plan.nsplit > 65535) return -5;
  const dim3 g1(static_cast<unsigned>(groups), static_cast<unsigned>(plan.nsplit));
  const bool vecR = aligned16(a.R) && (K % 8 == 0);
  const bool alignW = aligned16(a.hc_fn);
  cudaError_t e;
  if (a.T <= kKlMaxTokens && plan.KS <= 256 * kKlPer) {
    e = alignW ? launch_pdl(pre_cc_partial_klane_kernel<true>, g1, dim3(256), 0, s, a.R, a.hc_fn,
                            part, a.T, K, plan.KS)
               : launch_pdl(pre_cc_partial_klane_kernel<false>, g1, dim3(256), 0, s, a.R, a.hc_fn,
                            part, a.T, K, plan.KS);
  } else if (a.T <= kCcTokens && plan.KS <= kStMaxKS) {
    if (vecR && alignW)
      e = launch_pdl(pre_cc_partial_staged_kernel<true, true>, g1, dim3(256), 0, s, a.R, a.hc_fn,
                     part, a.T, K, plan.KS);
    else if (vecR)
      e = launch_pdl(pre_cc_partial_staged_kernel<true, false>, g1, dim3(256), 0, s, a.R, a.hc_fn,
                     part, a.T, K, plan.KS);
    else if (alignW)
      e = launch_pdl(pre_cc_partial_staged_kernel<false, true>, g1, dim3(256), 0, s, a.R, a.hc_fn,
                     part, a.T, K, plan.KS);
    else
      e = launch_pdl(pre_cc_partial_staged_kernel<false, false>, g1, dim3(256), 0, s, a.R,
                     a.hc_fn, part, a.T, K, plan.KS);
  } else if (vecR && alignW)
    e = launch_pdl(pre_cc_partial_kernel<true, true>, g1, dim3(256), 0, s, a.R,
                   a.hc_fn, part, a.T, K, plan.KS);
  else if (vecR)
    e = launch_pdl(pre_cc_partial_kernel<true, false>, g1, dim3(256), 0, s, a.R,
                   a.hc_fn, part, a.T, K, plan.KS);
  else if (alignW)
    e = launch_pdl(pre_cc_partial_kernel<false, true>, g1, dim3(256), 0, s, a.R,
                   a.hc_fn, part, a.T, K, plan.KS);
  else
    e = launch_pdl(pre_cc_partial_kernel<false, false>, g1, dim3(256), 0, s, a.R,
                   a.hc_fn, part, a.T, K, plan.KS);
  note_launches(1);
  if (e != cudaSuccess) return -4;
  *part_out = part;
  *nrec_out = static_cast<int>(plan.nsplit);
  return 0;
}

int launch_pre_cc(const PreArgs& a, cudaStream_t s) {
  const CcPlan plan = cc_plan(a.T, a.H);
  float* part = nullptr;
  int nrec = 0;
  const int r = launch_cc_projection(a, s, &part, &nrec);
  if (r != 0) return r;

  const int64_t nhb = (a.H + kAggCols - 1) / kAggCols;
  if (a.T > 0x7fffffff || 1 + nhb > 65535) return -5;
  const dim3 g2(static_cast<unsigned>(a.T), static_cast<unsigned>(1 + nhb));
  const FinishParams fp{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};
  const bool vec = aligned16(a.R) && aligned16(a.y) && (a.H % 8 == 0);
  cudaError_t e;
  if (vec)
    e = launch_pdl(pre_cc_finish_kernel<true>, g2, dim3(256), 0, s, a.R, part, plan.nsplit,
                   a.hc_scale, a.hc_base, a.y, a.pre, a.post, a.comb, a.T, a.H, fp);
  else
    e = launch_pdl(pre_cc_finish_kernel<false>, g2, dim3(256), 0, s, a.R, part, plan.nsplit,
                   a.hc_scale, a.hc_base, a.y, a.pre, a.post, a.comb, a.T, a.H, fp);
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

}  // namespace mhc
