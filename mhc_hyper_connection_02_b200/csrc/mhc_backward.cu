// Backward passes of the post-map and the pre-map: the exact derivatives of the forward
// definitions ("FlashInfer mHC module deep dive" §2.1 post-map, §3.4 / §5.2 pre-map; rwkv-ops
// mhu_jax.py names these backward kernels -- _mhc_post_op_ffi_bwd and mhc_pre_op's VJP -- without
// formulas).
//
// post-map  d_x = sum_n post[n] d_out[n];  d_R[o] = sum_n comb[o][n] d_out[n];
//           d_post[n] = sum_h x d_out[n];  d_comb[o][n] = sum_h R[o] d_out[n].
//           H >= 1024 (aligned, H % 8 == 0): persistent CTAs over tokens, the rows staged by bulk
//           copies into a shared-memory ring; otherwise one CTA per token with 16-byte (or
//           scalar) loads. Both: per-thread partial sums of the 20 coefficient gradients, a
//           fixed-order block reduction.
// pre-map   (upstream d_y, d_pre, d_post, d_comb; any may be absent)
//   1. the projection is recomputed by the forward's own kernels (records of raw and ss);
//   2. d_pre += sum_h d_y R_i: with the tensor projection (H % 64 == 0) the projection kernel forms
//      it from the R tiles it streams anyway (record floats 28..31), else one CTA per token;
//   3. per token (lane quad): rstd, logits, gates, the Sinkhorn forward (states checkpointed)
//      and the reverse pass -> d_raw, d_ss, the gates, and the per-token terms of d_scale, d_base;
//   4. d_scale, d_base: fixed-order sums over tokens;
//   5. d_R = d_raw . hc_fn^T + 2 R d_ss + pre_i d_y: on tcgen05 tensor cores where H % 128 == 0
//      (mhc_backward_tc.cu, with d_hc_fn in the same pass over R), else column slice x token
//      chunk per CTA, a thread's hc_fn weights in registers, fp32 on CUDA cores;
//   6. d_hc_fn = R_flat^T d_raw, where step 5 did not form it: on tcgen05 where 4H % 128 == 0
//      (mhc_backward_tc.cu: R read MN-major as the A operand), else column slice x token chunk
//      per CTA on CUDA cores; the partials are summed in order.
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kBwThreads = 256;

// Warp sum of v (fixed xor tree) into red[slot * 8 + warp]; the caller adds the 8 warps in order
// after a barrier.
__device__ __forceinline__ void bw_warp_partial(float v, float* red, int slot) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) red[slot * 8 + warp] = v;
}

// ------------------------------------------------------------------------------ post backward

template <bool kVec>
__global__ void __launch_bounds__(kBwThreads, 2) post_bwd_kernel(
    const uint16_t* __restrict__ dout, const uint16_t* __restrict__ x,
    const uint16_t* __restrict__ R, const float* __restrict__ post,
    const float* __restrict__ comb, uint16_t* __restrict__ dx, uint16_t* __restrict__ dR,
    float* __restrict__ dpost, float* __restrict__ dcomb, int64_t H) {
  __shared__ float red[20 * 8];
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  float p[4], c[4][4];
#pragma unroll
  for (int n = 0; n < 4; ++n) p[n] = __ldg(post + t * 4 + n);
#pragma unroll
  for (int o = 0; o < 4; ++o)
#pragma unroll
    for (int n = 0; n < 4; ++n) c[o][n] = __ldg(comb + t * 16 + o * 4 + n);
  float ap[4] = {0.f, 0.f, 0.f, 0.f}, ac[4][4];
#pragma unroll
  for (int o = 0; o < 4; ++o)
#pragma unroll
    for (int n = 0; n < 4; ++n) ac[o][n] = 0.f;
  const uint16_t* dO = dout + t * 4 * H;
  const uint16_t* Rt = R + t * 4 * H;
  const uint16_t* xt = x + t * H;
  if (kVec) {
    for (int64_t v = tid; v < H / 8; v += kBwThreads) {
      uint4 gv[4], rv[4];
#pragma unroll
      for (int n = 0; n < 4; ++n) gv[n] = ld_stream_ro(dO + n * H + v * 8);
#pragma unroll
      for (int o = 0; o < 4; ++o) rv[o] = ld_stream_ro(Rt + o * H + v * 8);
      const uint4 xv = ld_stream_ro(xt + v * 8);
      uint32_t ox[4], orr[4][4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        float g[2][4], r[2][4], xx[2];
#pragma unroll
        for (int n = 0; n < 4; ++n) {
          const uint32_t w = (&gv[n].x)[q];
          g[0][n] = bf16_lo(w);
          g[1][n] = bf16_hi(w);
        }
#pragma unroll
        for (int o = 0; o < 4; ++o) {
          const uint32_t w = (&rv[o].x)[q];
          r[0][o] = bf16_lo(w);
          r[1][o] = bf16_hi(w);
        }
        xx[0] = bf16_lo((&xv.x)[q]);
        xx[1] = bf16_hi((&xv.x)[q]);
        float vx[2], vr[2][4];
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float s = p[0] * g[e][0];
#pragma unroll
          for (int n = 1; n < 4; ++n) s = fmaf(p[n], g[e][n], s);
          vx[e] = s;
#pragma unroll
          for (int o = 0; o < 4; ++o) {
            float u = c[o][0] * g[e][0];
#pragma unroll
            for (int n = 1; n < 4; ++n) u = fmaf(c[o][n], g[e][n], u);
            vr[e][o] = u;
          }
#pragma unroll
          for (int n = 0; n < 4; ++n) {
            ap[n] = fmaf(xx[e], g[e][n], ap[n]);
#pragma unroll
            for (int o = 0; o < 4; ++o) ac[o][n] = fmaf(r[e][o], g[e][n], ac[o][n]);
          }
        }
        ox[q] = pack_bf16x2(vx[0], vx[1]);
#pragma unroll
        for (int o = 0; o < 4; ++o) orr[o][q] = pack_bf16x2(vr[0][o], vr[1][o]);
      }
      st_plain(dx + t * H + v * 8, make_uint4(ox[0], ox[1], ox[2], ox[3]));
#pragma unroll
      for (int o = 0; o < 4; ++o)
        st_plain(dR + t * 4 * H + o * H + v * 8,
                 make_uint4(orr[o][0], orr[o][1], orr[o][2], orr[o][3]));
    }
  } else {
    for (int64_t h = tid; h < H; h += kBwThreads) {
      float g[4], r[4];
#pragma unroll
      for (int n = 0; n < 4; ++n) g[n] = bf16_to_f32(dO[n * H + h]);
#pragma unroll
      for (int o = 0; o < 4; ++o) r[o] = bf16_to_f32(Rt[o * H + h]);
      const float xx = bf16_to_f32(xt[h]);
      float s = p[0] * g[0];
#pragma unroll
      for (int n = 1; n < 4; ++n) s = fmaf(p[n], g[n], s);
      dx[t * H + h] = f32_to_bf16(s);
#pragma unroll
      for (int o = 0; o < 4; ++o) {
        float u = c[o][0] * g[0];
#pragma unroll
        for (int n = 1; n < 4; ++n) u = fmaf(c[o][n], g[n], u);
        dR[t * 4 * H + o * H + h] = f32_to_bf16(u);
      }
#pragma unroll
      for (int n = 0; n < 4; ++n) {
        ap[n] = fmaf(xx, g[n], ap[n]);
#pragma unroll
        for (int o = 0; o < 4; ++o) ac[o][n] = fmaf(r[o], g[n], ac[o][n]);
      }
    }
  }
  // Block sums of the 20 coefficient gradients, fixed order (xor tree in each warp, then warps).
#pragma unroll
  for (int n = 0; n < 4; ++n) bw_warp_partial(ap[n], red, n);
#pragma unroll
  for (int o = 0; o < 4; ++o)
#pragma unroll
    for (int n = 0; n < 4; ++n) bw_warp_partial(ac[o][n], red, 4 + o * 4 + n);
  __syncthreads();
  if (tid < 20) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[tid * 8 + w];
    if (tid < 4)
      dpost[t * 4 + tid] = s;
    else
      dcomb[t * 16 + (tid - 4)] = s;
  }
}

// Persistent form (H % 8 == 0, 16-byte aligned rows): CTA j takes tokens j, j + P, .... For each,
// one producer thread stages the token's nine input rows (d_out[0..3], R[0..3], x) chunk by chunk
// (1024 columns, 18 KB) into a four-stage shared-memory ring with 1-D bulk copies completing on an
// mbarrier; 128 consumer threads take 8 columns each, write d_x and d_R straight to global and
// carry their partial sums of the 20 coefficient gradients across the token's chunks, which end
// in a fixed-order reduction (xor tree within each warp, then the four warps in order). Three
// CTAs per SM keep 216 KB of loads in flight (measured against two CTAs of five or six stages:
// 282.6 us against 287-290 us at T=8192, H=7168). All waits are bounded.
constexpr int kPbChunk = 1024;
constexpr int kPbStages = 4;
constexpr int kPbConsumers = kPbChunk / 8;                 // 128
constexpr int kPbThreads = kPbConsumers + 32;              // + one producer warp
constexpr int kPbRows = 9;
constexpr int kPbCtas = 3;                                 // per SM: 3 x 72 KB of stages
constexpr int kPbStageBytes = kPbRows * kPbChunk * 2;      // 18 KB
constexpr int kPbSmem = kPbStages * kPbStageBytes + 2 * kPbStages * 8 + 4 * 20 * 4;

__global__ void __launch_bounds__(kPbThreads, kPbCtas) post_bwd_persistent_kernel(
    const uint16_t* __restrict__ dout, const uint16_t* __restrict__ x,
    const uint16_t* __restrict__ R, const float* __restrict__ post,
    const float* __restrict__ comb, uint16_t* __restrict__ dx, uint16_t* __restrict__ dR,
    float* __restrict__ dpost, float* __restrict__ dcomb, int64_t T, int64_t H) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* stage_base = reinterpret_cast<uint16_t*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPbStages * kPbStageBytes);
  uint64_t* empty = full + kPbStages;
  float* red = reinterpret_cast<float*>(empty + kPbStages);  // [4 warps][20]
  const int64_t chunks = (H + kPbChunk - 1) / kPbChunk;
  const int tid = threadIdx.x;

  if (tid == 0) {
    for (int st = 0; st < kPbStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], kPbConsumers);
    }
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait();
  pdl_trigger();

  if (tid >= kPbConsumers) {
    // Producer warp: lane 0 issues the copies.
    if (tid == kPbConsumers) {
      int st = 0;
      uint32_t phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int64_t t = blockIdx.x; t < T && ok; t += gridDim.x) {
        for (int64_t c = 0; c < chunks; ++c) {
          if (issued >= kPbStages && !mbar_wait(&empty[st], phase ^ 1u, 120)) {
            ok = false;
            break;
          }
          const int64_t h0 = c * kPbChunk;
          const uint32_t bytes = static_cast<uint32_t>(
              (H - h0 < kPbChunk ? H - h0 : static_cast<int64_t>(kPbChunk)) * 2);
          uint16_t* sb = stage_base + st * (kPbRows * kPbChunk);
          mbar_arrive_expect_tx(&full[st], kPbRows * bytes);
#pragma unroll
          for (int n = 0; n < 4; ++n)
            bulk_g2s(sb + n * kPbChunk, dout + (t * 4 + n) * H + h0, bytes, &full[st]);
#pragma unroll
          for (int o = 0; o < 4; ++o)
            bulk_g2s(sb + (4 + o) * kPbChunk, R + (t * 4 + o) * H + h0, bytes, &full[st]);
          bulk_g2s(sb + 8 * kPbChunk, x + t * H + h0, bytes, &full[st]);
          ++issued;
          if (++st == kPbStages) {
            st = 0;
            phase ^= 1u;
          }
        }
      }
      // Do not leave the CTA while copies into its shared memory are in flight: stage i was
      // filled n_i times, its last fill completes the phase with parity (n_i - 1) & 1.
      if (!ok) {
        for (int i = 0; i < kPbStages; ++i) {
          const int64_t n_i = issued / kPbStages + (i < issued % kPbStages ? 1 : 0);
          if (n_i > 0) mbar_wait(&full[i], static_cast<uint32_t>((n_i - 1) & 1), 122);
        }
      }
    }
    return;
  }

  // Consumers: thread tid owns columns h0 + 8 tid .. + 8 of every chunk.
  const int lane = tid & 31, warp = tid >> 5;
  int st = 0;
  uint32_t phase = 0;
  bool ok = true;
  for (int64_t t = blockIdx.x; t < T; t += gridDim.x) {
    float p[4], cm[4][4];
#pragma unroll
    for (int n = 0; n < 4; ++n) p[n] = __ldg(post + t * 4 + n);
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int n = 0; n < 4; ++n) cm[o][n] = __ldg(comb + t * 16 + o * 4 + n);
    float ap[4] = {0.f, 0.f, 0.f, 0.f}, ac[4][4];
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int n = 0; n < 4; ++n) ac[o][n] = 0.f;
    for (int64_t c = 0; c < chunks; ++c) {
      ok = __all_sync(0xffffffffu, mbar_wait(&full[st], phase, 121));
      if (!ok) break;
      const int64_t h0 = c * kPbChunk;
      const int64_t n = H - h0 < kPbChunk ? H - h0 : static_cast<int64_t>(kPbChunk);
      const uint16_t* sb = stage_base + st * (kPbRows * kPbChunk);
      const int e = tid * 8;
      if (e < n) {
        uint4 gv[4], rv[4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          gv[q] = *reinterpret_cast<const uint4*>(sb + q * kPbChunk + e);
          rv[q] = *reinterpret_cast<const uint4*>(sb + (4 + q) * kPbChunk + e);
        }
        const uint4 xv = *reinterpret_cast<const uint4*>(sb + 8 * kPbChunk + e);
        uint32_t ox[4], orr[4][4];
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          float g[2][4], r[2][4], xx[2];
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            const uint32_t w = (&gv[m].x)[q];
            g[0][m] = bf16_lo(w);
            g[1][m] = bf16_hi(w);
          }
#pragma unroll
          for (int o = 0; o < 4; ++o) {
            const uint32_t w = (&rv[o].x)[q];
            r[0][o] = bf16_lo(w);
            r[1][o] = bf16_hi(w);
          }
          xx[0] = bf16_lo((&xv.x)[q]);
          xx[1] = bf16_hi((&xv.x)[q]);
          float vx[2], vr[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            float sx = p[0] * g[u][0];
#pragma unroll
            for (int m = 1; m < 4; ++m) sx = fmaf(p[m], g[u][m], sx);
            vx[u] = sx;
#pragma unroll
            for (int o = 0; o < 4; ++o) {
              float sr = cm[o][0] * g[u][0];
#pragma unroll
              for (int m = 1; m < 4; ++m) sr = fmaf(cm[o][m], g[u][m], sr);
              vr[u][o] = sr;
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
              ap[m] = fmaf(xx[u], g[u][m], ap[m]);
#pragma unroll
              for (int o = 0; o < 4; ++o) ac[o][m] = fmaf(r[u][o], g[u][m], ac[o][m]);
            }
          }
          ox[q] = pack_bf16x2(vx[0], vx[1]);
#pragma unroll
          for (int o = 0; o < 4; ++o) orr[o][q] = pack_bf16x2(vr[0][o], vr[1][o]);
        }
        st_stream(dx + t * H + h0 + e, make_uint4(ox[0], ox[1], ox[2], ox[3]));
#pragma unroll
        for (int o = 0; o < 4; ++o)
          st_stream(dR + (t * 4 + o) * H + h0 + e,
                    make_uint4(orr[o][0], orr[o][1], orr[o][2], orr[o][3]));
      }
      mbar_arrive(&empty[st]);
      if (++st == kPbStages) {
        st = 0;
        phase ^= 1u;
      }
    }
    // The four consumer warps agree on going on (a stop keeps the barrier sequence matched).
    if (named_bar_or(1, kPbConsumers, !ok)) return;
#pragma unroll
    for (int m = 0; m < 4; ++m) {
      float v = ap[m];
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp * 20 + m] = v;
    }
#pragma unroll
    for (int o = 0; o < 4; ++o)
#pragma unroll
      for (int m = 0; m < 4; ++m) {
        float v = ac[o][m];
#pragma unroll
        for (int k = 16; k > 0; k >>= 1) v += __shfl_xor_sync(0xffffffffu, v, k);
        if (lane == 0) red[warp * 20 + 4 + o * 4 + m] = v;
      }
    named_bar_or(1, kPbConsumers, false);
    if (tid < 20) {
      const float v = ((red[tid] + red[20 + tid]) + red[40 + tid]) + red[60 + tid];
      if (tid < 4)
        dpost[t * 4 + tid] = v;
      else
        dcomb[t * 16 + (tid - 4)] = v;
    }
    named_bar_or(1, kPbConsumers, false);  // red is read before the next token overwrites it
  }
}

int launch_post_backward(const uint16_t* dout, const uint16_t* x, const uint16_t* R,
                         const float* post, const float* comb, uint16_t* dx, uint16_t* dR,
                         float* dpost, float* dcomb, int64_t T, int64_t H, cudaStream_t s) {
  if (T > 0x7fffffff) return -5;
  const bool vec = H % 8 == 0 && aligned16(dout) && aligned16(x) && aligned16(R) &&
                   aligned16(dx) && aligned16(dR);
  // Rows of at least one full chunk: the persistent bulk-copy form.
  if (vec && H >= kPbChunk &&
      ensure_smem_limit(reinterpret_cast<const void*>(post_bwd_persistent_kernel), kPbSmem)) {
    int64_t blocks = kPbCtas * static_cast<int64_t>(device_sm_count());
    if (blocks > T) blocks = T;
    if (launch_pdl(post_bwd_persistent_kernel, dim3(static_cast<unsigned>(blocks)),
                   dim3(kPbThreads), static_cast<size_t>(kPbSmem), s, dout, x, R, post, comb, dx,
                   dR, dpost, dcomb, T, H) != cudaSuccess)
      return -4;
    note_launches(1);
    return 0;
  }
  const cudaError_t e =
      vec ? launch_pdl(post_bwd_kernel<true>, dim3(static_cast<unsigned>(T)), dim3(kBwThreads), 0,
                       s, dout, x, R, post, comb, dx, dR, dpost, dcomb, H)
          : launch_pdl(post_bwd_kernel<false>, dim3(static_cast<unsigned>(T)), dim3(kBwThreads),
                       0, s, dout, x, R, post, comb, dx, dR, dpost, dcomb, H);
  if (e != cudaSuccess) return -4;
  note_launches(1);
  return 0;
}


// ------------------------------------------------------------------------------ pre backward

constexpr int kBrec = 64;  // floats per token of the backward record (see pre_bwd_coef_kernel)

// d_pre_tot[t][i] = d_pre[t][i] + sum_h d_y[t][h] R[t][i][h] (d_pre, d_y may be null).
template <bool kVec>
__global__ void __launch_bounds__(kBwThreads) pre_bwd_dpre_kernel(
    const uint16_t* __restrict__ dy, const float* __restrict__ dpre,
    const uint16_t* __restrict__ R, float* __restrict__ dpt, int64_t H) {
  __shared__ float red[4 * 8];
  const int64_t t = blockIdx.x;
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (dy) {
    const uint16_t* Rt = R + t * 4 * H;
    const uint16_t* gt = dy + t * H;
    if (kVec) {
      for (int64_t v = tid; v < H / 8; v += kBwThreads) {
        const uint4 g = ld_stream_ro(gt + v * 8);
        uint4 rv[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) rv[i] = ld_stream_ro(Rt + i * H + v * 8);
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const float g0 = bf16_lo((&g.x)[q]), g1 = bf16_hi((&g.x)[q]);
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            a[i] = fmaf(g0, bf16_lo((&rv[i].x)[q]), a[i]);
            a[i] = fmaf(g1, bf16_hi((&rv[i].x)[q]), a[i]);
          }
        }
      }
    } else {
      for (int64_t h = tid; h < H; h += kBwThreads) {
        const float g = bf16_to_f32(gt[h]);
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = fmaf(g, bf16_to_f32(Rt[i * H + h]), a[i]);
      }
    }
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) bw_warp_partial(a[i], red, i);
  __syncthreads();
  if (tid < 4) {
    float s = dpre ? dpre[t * 4 + tid] : 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[tid * 8 + w];
    dpt[t * 4 + tid] = s;
  }
}

__device__ __forceinline__ float quad_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v + __shfl_xor_sync(0xffffffffu, v, 2);
}

// One Sinkhorn round on the quad's 4x4 (lane r holds row r): row normalisation then column
// normalisation by plain sums, with the forward's arithmetic (sinkhorn_quad: multiplication by
// recip_nr of the sum, column sums (a0 + a1) + (a2 + a3) across the quad), so the recomputed
// states are the forward's bit for bit; returns B (after the row step) and the reciprocals of the
// normalisers for the reverse pass.
__device__ __forceinline__ void sk_round(float (&a)[4], float (&b)[4], float& rrs,
                                         float (&rcs)[4]) {
  rrs = recip_nr(((a[0] + a[1]) + a[2]) + a[3]);
#pragma unroll
  for (int n = 0; n < 4; ++n) b[n] = a[n] * rrs;
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    float c = b[n] + __shfl_xor_sync(0xffffffffu, b[n], 1);
    c = c + __shfl_xor_sync(0xffffffffu, c, 2);
    rcs[n] = recip_nr(c);
    a[n] = b[n] * rcs[n];
  }
}

constexpr int kSkCk = 32;  // Sinkhorn forward checkpoints kept by the reverse pass (every round up to 32)

// Per token, one lane quad (lane r: pre r, post r, comb row r). Writes the backward record
// brec[t][64]: [0..23] d_raw, [24] d_ss, [25..28] pre gates, [29..31] the token's terms of
// d_scale, [32..55] d_l (the token's term of d_base).
__global__ void __launch_bounds__(256) pre_bwd_coef_kernel(
    const float* __restrict__ part, int nrec, const float* __restrict__ dpt,
    const float* __restrict__ dpre_in, int dp_in_records,
    const float* __restrict__ dpost, const float* __restrict__ dcomb,
    const float* __restrict__ scale, const float* __restrict__ base, float* __restrict__ brec,
    int64_t T, int64_t K, FinishParams fp) {
  const int lane = threadIdx.x & 31;
  const int r = lane & 3;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 2;
  const bool live = t < T;
  const int64_t tt = live ? t : 0;
  pdl_wait();
  pdl_trigger();
  float g0 = 0.f, g1 = 0.f, gc[4] = {0.f, 0.f, 0.f, 0.f}, ss = 0.f, dy_r = 0.f;
  for (int s = 0; s < nrec; ++s) {
    const float* rec = part + (static_cast<int64_t>(s) * T + tt) * 32;
    g0 += __ldg(rec + r);
    g1 += __ldg(rec + 4 + r);
#pragma unroll
    for (int n = 0; n < 4; ++n) gc[n] += __ldg(rec + 8 + 4 * r + n);
    ss += __ldg(rec + 24);
    if (dp_in_records) dy_r += __ldg(rec + 28 + r);  // sum_h d_y R_r, formed with the projection
  }
  const float rstd = 1.0f / sqrtf(ss / static_cast<float>(K) + fp.rms_eps);
  const float s0 = __ldg(scale), s1 = __ldg(scale + 1), s2 = __ldg(scale + 2);
  const float m0 = g0 * rstd, m1 = g1 * rstd;
  float mc[4], lc[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) {
    mc[n] = gc[n] * rstd;
    lc[n] = fmaf(mc[n], s2, __ldg(base + 8 + 4 * r + n));
  }
  const float sg0 = 1.0f / (1.0f + expf(-fmaf(m0, s0, __ldg(base + r))));
  const float sg1 = 1.0f / (1.0f + expf(-fmaf(m1, s1, __ldg(base + 4 + r))));
  const float dpr = dp_in_records ? (dpre_in ? dpre_in[tt * 4 + r] : 0.f) + dy_r : dpt[tt * 4 + r];
  const float dl0 = dpr * sg0 * (1.0f - sg0);
  const float dl1 = (dpost ? dpost[tt * 4 + r] : 0.f) * fp.post_mult * sg1 * (1.0f - sg1);

  // Sinkhorn reverse pass. The forward starts from P = softmax(row) and A0 = P + eps; its states
  // are checkpointed every G rounds (at most kSkCk checkpoints); the state entering round k is
  // recomputed from the checkpoint at or before it, by the same operations as the forward, so it
  // is the forward's state exactly.
  float p[4], a0[4], dA[4];
  {
    const float mx = fmaxf(fmaxf(lc[0], lc[1]), fmaxf(lc[2], lc[3]));
    float e[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) e[n] = expf(lc[n] - mx);
    const float res = recip_nr(((e[0] + e[1]) + e[2]) + e[3]);
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      p[n] = e[n] * res;
      a0[n] = fmaf(e[n], res, fp.sinkhorn_eps);  // as the forward forms A0
      dA[n] = dcomb ? dcomb[tt * 16 + 4 * r + n] : 0.f;
    }
  }
  const int G = (fp.iters + kSkCk - 1) / kSkCk;
  float ck[kSkCk][4];
  {
    float a[4] = {a0[0], a0[1], a0[2], a0[3]}, b[4], rrs, rcs[4];
    for (int k = 0; k < fp.iters; ++k) {
      if (k % G == 0) {
#pragma unroll
        for (int n = 0; n < 4; ++n) ck[k / G][n] = a[n];
      }
      sk_round(a, b, rrs, rcs);
    }
  }
  for (int k = fp.iters - 1; k >= 0; --k) {
    const int c = k / G;
    float a[4] = {ck[c][0], ck[c][1], ck[c][2], ck[c][3]}, b[4], rrs, rcs[4];
    for (int j = c * G; j < k; ++j) sk_round(a, b, rrs, rcs);
    sk_round(a, b, rrs, rcs);  // round k: a is now C
    float dB[4];
#pragma unroll
    for (int n = 0; n < 4; ++n) dB[n] = (dA[n] - quad_sum(dA[n] * a[n])) * rcs[n];
    const float rdot = ((dB[0] * b[0] + dB[1] * b[1]) + dB[2] * b[2]) + dB[3] * b[3];
#pragma unroll
    for (int n = 0; n < 4; ++n) dA[n] = (dB[n] - rdot) * rrs;
  }
  // Softmax: d_l = P (dA0 - sum_n dA0 P) along the row.
  float dlc[4];
  {
    const float pd = ((dA[0] * p[0] + dA[1] * p[1]) + dA[2] * p[2]) + dA[3] * p[3];
#pragma unroll
    for (int n = 0; n < 4; ++n) dlc[n] = p[n] * (dA[n] - pd);
  }

  const float dm0 = dl0 * s0, dm1 = dl1 * s1;
  float dmc[4];
#pragma unroll
  for (int n = 0; n < 4; ++n) dmc[n] = dlc[n] * s2;
  float drs = fmaf(dm0, g0, dm1 * g1);
#pragma unroll
  for (int n = 0; n < 4; ++n) drs = fmaf(dmc[n], gc[n], drs);
  const float d_rstd = quad_sum(drs);
  const float d_ss = -0.5f * rstd * rstd * rstd / static_cast<float>(K) * d_rstd;
  const float sc0 = quad_sum(dl0 * m0), sc1 = quad_sum(dl1 * m1);
  float scc = 0.f;
#pragma unroll
  for (int n = 0; n < 4; ++n) scc = fmaf(dlc[n], mc[n], scc);
  scc = quad_sum(scc);
  if (live) {
    float* o = brec + t * kBrec;
    o[r] = dm0 * rstd;
    o[4 + r] = dm1 * rstd;
#pragma unroll
    for (int n = 0; n < 4; ++n) o[8 + 4 * r + n] = dmc[n] * rstd;
    o[25 + r] = sg0 + fp.pre_eps;
    o[32 + r] = dl0;
    o[36 + r] = dl1;
#pragma unroll
    for (int n = 0; n < 4; ++n) o[40 + 4 * r + n] = dlc[n];
    if (r == 0) {
      o[24] = d_ss;
      o[29] = sc0;
      o[30] = sc1;
      o[31] = scc;
    }
  }
}

// d_scale[g] = sum_t brec[t][29 + g]; d_base[j] = sum_t brec[t][32 + j]: block b sums column b in a
// fixed order (strided per thread, then a fixed tree).
__global__ void __launch_bounds__(256) pre_bwd_param_kernel(const float* __restrict__ brec,
                                                            float* __restrict__ dscale,
                                                            float* __restrict__ dbase, int64_t T) {
  __shared__ float red[8];
  const int b = blockIdx.x;  // 0..26
  const int col = b < 3 ? 29 + b : 32 + (b - 3);
  pdl_wait();
  pdl_trigger();
  float v = 0.f;
  for (int64_t t = threadIdx.x; t < T; t += blockDim.x) v += brec[t * kBrec + col];
  bw_warp_partial(v, red, 0);
  __syncthreads();
  if (threadIdx.x == 0) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < 8; ++w) s += red[w];
    if (b < 3)
      dscale[b] = s;
    else
      dbase[b - 3] = s;
  }
}

// 16-byte and 4-byte asynchronous copies global -> shared for the contraction kernels' staging.
__device__ __forceinline__ void bw_cp16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void bw_cp_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void bw_cp_wait() {  // all but the N newest groups have landed
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

constexpr int kDxThreads = 128;
constexpr int kDxCols = 4 * kDxThreads;  // columns of the flattened row per CTA
constexpr int kDxTok = 12;               // tokens per staged step (two buffers)
constexpr int kDxSmem = 2 * kDxTok * (2 * kDxCols * 2 + 32 * 4);  // R, d_y tiles + records
constexpr int kDxSlotsPerSm = 4;  // resident CTAs per SM (shared memory) the chunking aims at

// d_R = d_raw . hc_fn^T + 2 R d_ss + pre_i d_y over a slice of kDxCols columns and a chunk of
// tokens. A thread holds hc_fn's 24 weights of its 4 columns in registers and runs through the
// chunk's tokens; each step's R and d_y tiles [kDxTok][kDxCols] and the tokens' records (d_raw,
// d_ss, pre) are staged in shared memory by asynchronous copies one step ahead. Per element the
// arithmetic is acc = sum_j d_raw[j] w[j] in j order from 0, then fma(pre_i, dy, fma(2 d_ss, R,
// acc)), rounded once. Requires H % 8 == 0 and 16-byte aligned R, d_R, d_y.
__global__ void __launch_bounds__(kDxThreads, kDxSlotsPerSm) pre_bwd_dx_kernel(
    const uint16_t* __restrict__ R, const uint16_t* __restrict__ dy,
    const float* __restrict__ W, const float* __restrict__ brec, uint16_t* __restrict__ dR,
    int64_t T, int64_t H, int64_t tchunk) {
  extern __shared__ __align__(16) uint8_t dx_smem[];
  uint16_t* xs = reinterpret_cast<uint16_t*>(dx_smem);      // [2][kDxTok][kDxCols]
  uint16_t* gs = xs + 2 * kDxTok * kDxCols;                 // [2][kDxTok][kDxCols]
  float* tv = reinterpret_cast<float*>(gs + 2 * kDxTok * kDxCols);  // [2][kDxTok][32]
  const int64_t K = 4 * H;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kDxCols;
  const int tid = threadIdx.x;
  const int64_t kb = k0 + 4 * tid;  // this thread's 4 columns (K % 4 == 0)
  const bool kvalid = kb < K;
  const int64_t si = kvalid ? kb / H : 0;
  const int64_t tb = static_cast<int64_t>(blockIdx.y) * tchunk;
  const int64_t te = min(T, tb + tchunk);
  pdl_wait();
  pdl_trigger();
  float w[4][kMix];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int j = 0; j < kMix; ++j) w[c][j] = kvalid ? __ldg(W + (kb + c) * kMix + j) : 0.f;

  const int nsteps = static_cast<int>((te - tb + kDxTok - 1) / kDxTok);
  // Staging: this thread always copies 8-column chunk sc of the slice, for tokens sr + 2 u.
  static_assert(kDxThreads == 2 * (kDxCols / 8), "staging map");
  const int sc = tid & (kDxCols / 8 - 1), sr = tid / (kDxCols / 8);
  const int64_t sk = k0 + sc * 8;
  const bool skv = sk < K;
  const int64_t sh = skv ? sk - (sk / H) * H : 0;  // d_y column of the chunk
  auto stage = [&](int step, int b) {
    const int64_t t0 = tb + static_cast<int64_t>(step) * kDxTok;
    if (skv) {
      const uint16_t* rp = R + (t0 + sr) * K + sk;
      const uint16_t* gp = dy ? dy + (t0 + sr) * H + sh : nullptr;
      uint16_t* xd = xs + (b * kDxTok + sr) * kDxCols + sc * 8;
      uint16_t* gd = gs + (b * kDxTok + sr) * kDxCols + sc * 8;
#pragma unroll
      for (int u = 0; u < kDxTok / 2; ++u) {
        if (t0 + sr + 2 * u < te) {
          bw_cp16(xd + 2 * u * kDxCols, rp + 2 * u * K);
          if (gp) bw_cp16(gd + 2 * u * kDxCols, gp + 2 * u * H);
        }
      }
    }
    for (int e = tid; e < kDxTok * 8; e += kDxThreads) {  // record floats 0..31 of each token
      const int tl = e >> 3, q = e & 7;
      const int64_t t = t0 + tl;
      if (t < te) bw_cp16(tv + (b * kDxTok + tl) * 32 + q * 4, brec + t * kBrec + q * 4);
    }
    bw_cp_commit();
  };
  if (nsteps > 0) stage(0, 0);
  for (int step = 0; step < nsteps; ++step) {
    const int b = step & 1;
    if (step + 1 < nsteps) {
      stage(step + 1, b ^ 1);
      bw_cp_wait<1>();
    } else {
      bw_cp_wait<0>();
    }
    __syncthreads();  // step's tiles visible to every thread
    const int64_t t0 = tb + static_cast<int64_t>(step) * kDxTok;
    const int n = static_cast<int>(min(static_cast<int64_t>(kDxTok), te - t0));
    if (kvalid) {
      for (int tl = 0; tl < n; ++tl) {
        const float* o = tv + (b * kDxTok + tl) * 32;
        float d[kMix];
#pragma unroll
        for (int q = 0; q < kMix / 4; ++q) {
          const float4 v = *reinterpret_cast<const float4*>(o + 4 * q);
          d[4 * q] = v.x;
          d[4 * q + 1] = v.y;
          d[4 * q + 2] = v.z;
          d[4 * q + 3] = v.w;
        }
        const float dss2 = 2.0f * o[24];
        const float pi = o[25 + si];
        const int off = (b * kDxTok + tl) * kDxCols + 4 * tid;
        const uint2 xv = *reinterpret_cast<const uint2*>(xs + off);
        const uint2 gv = dy ? *reinterpret_cast<const uint2*>(gs + off) : make_uint2(0u, 0u);
        float acc[4];
#pragma unroll
        for (int c = 0; c < 4; ++c) {
          acc[c] = 0.f;
#pragma unroll
          for (int j = 0; j < kMix; ++j) acc[c] = fmaf(d[j], w[c][j], acc[c]);
        }
        const float x0 = bf16_lo(xv.x), x1 = bf16_hi(xv.x), x2 = bf16_lo(xv.y), x3 = bf16_hi(xv.y);
        const float g0 = bf16_lo(gv.x), g1 = bf16_hi(gv.x), g2 = bf16_lo(gv.y), g3 = bf16_hi(gv.y);
        const uint32_t o0 = pack_bf16x2(fmaf(pi, g0, fmaf(dss2, x0, acc[0])),
                                        fmaf(pi, g1, fmaf(dss2, x1, acc[1])));
        const uint32_t o1 = pack_bf16x2(fmaf(pi, g2, fmaf(dss2, x2, acc[2])),
                                        fmaf(pi, g3, fmaf(dss2, x3, acc[3])));
        *reinterpret_cast<uint2*>(dR + (t0 + tl) * K + kb) = make_uint2(o0, o1);
      }
    }
    __syncthreads();  // buffer b is restaged two steps on
  }
}

// Any H / alignment: one thread per element of d_R.
__global__ void __launch_bounds__(256) pre_bwd_dx_scalar_kernel(
    const uint16_t* __restrict__ R, const uint16_t* __restrict__ dy,
    const float* __restrict__ W, const float* __restrict__ brec, uint16_t* __restrict__ dR,
    int64_t T, int64_t H) {
  const int64_t K = 4 * H;
  pdl_wait();
  pdl_trigger();
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < T * K;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = u / K, k = u - t * K;
    const float* o = brec + t * kBrec;
    float acc = 0.f;
#pragma unroll 4
    for (int j = 0; j < kMix; ++j) acc = fmaf(o[j], __ldg(W + k * kMix + j), acc);
    const int64_t i = k / H, h = k - i * H;
    acc = fmaf(2.0f * o[24], bf16_to_f32(R[u]), acc);
    if (dy) acc = fmaf(o[25 + i], bf16_to_f32(dy[t * H + h]), acc);
    dR[u] = f32_to_bf16(acc);
  }
}

constexpr int kDwThreads = 128;
constexpr int kDwCols = 4 * kDwThreads;  // columns of hc_fn per CTA
constexpr int kDwTok = 16;               // tokens per staged step (two buffers)
constexpr int kDwSlotsPerSm = 4;         // resident CTAs per SM the chunking aims at

// Partial d_hc_fn over a token chunk: dwp[chunk][k][j] = sum_{t in chunk} R_flat[t][k] d_raw[t][j],
// tokens in increasing order. A thread owns 4 columns x all 24 logits (96 accumulators); per
// token it reads its 4 bf16 values and the token's d_raw (a broadcast) from shared memory, where
// each step's R tile [kDwTok][kDwCols] (bf16, as stored) and d_raw rows are staged one step ahead
// (asynchronous 16-byte copies when kVec: H % 8 == 0 and R 16-byte aligned).
template <bool kVec>
__global__ void __launch_bounds__(kDwThreads, kDwSlotsPerSm)
    pre_bwd_dw_kernel(const uint16_t* __restrict__ R, const float* __restrict__ brec,
                      float* __restrict__ dwp, int64_t T, int64_t H, int64_t tchunk) {
  __shared__ __align__(16) uint16_t xs[2][kDwTok][kDwCols];
  __shared__ __align__(16) float ds[2][kDwTok][kMix];
  const int64_t K = 4 * H;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x) * kDwCols;
  const int64_t tb = static_cast<int64_t>(blockIdx.y) * tchunk;
  const int64_t te = min(T, tb + tchunk);
  const int tid = threadIdx.x;
  const int64_t kb = k0 + 4 * tid;
  pdl_wait();
  pdl_trigger();
  float acc[4][kMix];
#pragma unroll
  for (int c = 0; c < 4; ++c)
#pragma unroll
    for (int j = 0; j < kMix; ++j) acc[c][j] = 0.f;

  const int nsteps = static_cast<int>((te - tb + kDwTok - 1) / kDwTok);
  auto stage = [&](int step, int b) {
    const int64_t t0 = tb + static_cast<int64_t>(step) * kDwTok;
    if (kVec) {  // this thread copies 8-column chunk sc for tokens sr + 2 u
      static_assert(kDwThreads == 2 * (kDwCols / 8), "staging map");
      const int sc = tid & (kDwCols / 8 - 1), sr = tid / (kDwCols / 8);
      if (k0 + sc * 8 < K) {
        const uint16_t* rp = R + (t0 + sr) * K + k0 + sc * 8;
#pragma unroll
        for (int u = 0; u < kDwTok / 2; ++u)
          if (t0 + sr + 2 * u < te) bw_cp16(&xs[b][sr + 2 * u][sc * 8], rp + 2 * u * K);
      }
    } else {
      for (int e = tid; e < kDwTok * kDwCols; e += kDwThreads) {
        const int tl = e / kDwCols, c = e - tl * kDwCols;
        const int64_t t = t0 + tl, k = k0 + c;
        if (t < te && k < K) xs[b][tl][c] = R[t * K + k];
      }
    }
    for (int e = tid; e < kDwTok * (kMix / 4); e += kDwThreads) {  // d_raw: 6 x 16 bytes a token
      const int tl = e / (kMix / 4), q = e - tl * (kMix / 4);
      const int64_t t = t0 + tl;
      if (t < te) bw_cp16(&ds[b][tl][q * 4], brec + t * kBrec + q * 4);
    }
    bw_cp_commit();
  };
  if (nsteps > 0) stage(0, 0);
  for (int step = 0; step < nsteps; ++step) {
    const int b = step & 1;
    if (step + 1 < nsteps) {
      stage(step + 1, b ^ 1);
      bw_cp_wait<1>();
    } else {
      bw_cp_wait<0>();
    }
    __syncthreads();
    const int64_t t0 = tb + static_cast<int64_t>(step) * kDwTok;
    const int n = static_cast<int>(min(static_cast<int64_t>(kDwTok), te - t0));
    if (kb < K) {
      for (int tl = 0; tl < n; ++tl) {
        const uint2 xv = *reinterpret_cast<const uint2*>(&xs[b][tl][4 * tid]);
        const float xf[4] = {bf16_lo(xv.x), bf16_hi(xv.x), bf16_lo(xv.y), bf16_hi(xv.y)};
#pragma unroll
        for (int q = 0; q < kMix / 4; ++q) {
          const float4 d4 = *reinterpret_cast<const float4*>(&ds[b][tl][4 * q]);
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            acc[c][4 * q] = fmaf(xf[c], d4.x, acc[c][4 * q]);
            acc[c][4 * q + 1] = fmaf(xf[c], d4.y, acc[c][4 * q + 1]);
            acc[c][4 * q + 2] = fmaf(xf[c], d4.z, acc[c][4 * q + 2]);
            acc[c][4 * q + 3] = fmaf(xf[c], d4.w, acc[c][4 * q + 3]);
          }
        }
      }
    }
    __syncthreads();  // buffer b is restaged two steps on
  }
  if (kb < K) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float4* o = reinterpret_cast<float4*>(dwp + (static_cast<int64_t>(blockIdx.y) * K + kb + c) *
                                                      kMix);
#pragma unroll
      for (int q = 0; q < kMix / 4; ++q)
        o[q] = make_float4(acc[c][4 * q], acc[c][4 * q + 1], acc[c][4 * q + 2], acc[c][4 * q + 3]);
    }
  }
}

// d_hc_fn[k][j] = sum over chunks (in order) of the partials.
__global__ void __launch_bounds__(256) pre_bwd_dw_sum_kernel(const float* __restrict__ dwp,
                                                             float* __restrict__ dw, int64_t KJ,
                                                             int nchunk) {
  pdl_wait();
  pdl_trigger();
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < KJ;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    float s = 0.f;
    for (int c = 0; c < nchunk; ++c) s += dwp[c * KJ + u];
    dw[u] = s;
  }
}

struct BwPlan {
  size_t proj, dpt, brec, dwp, drtc, dwtc, total;
  int64_t tchunk;
  int nchunk;
};

static BwPlan bw_plan(int64_t T, int64_t H) {
  BwPlan p;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  size_t a = pre_tc_workspace_bytes(T, H), b = pre_cc_workspace_bytes(T, H);
  p.proj = up(a > b ? a : b);
  p.dpt = up(static_cast<size_t>(T) * 16);
  p.brec = up(static_cast<size_t>(T) * kBrec * 4);
  // Token chunks of d_hc_fn partials: column slices x chunks fill the SMs' CTA slots in one
  // wave (the same chunks serve d_R).
  const int64_t kcols = (4 * H + kDwCols - 1) / kDwCols;
  int64_t nchunk = (kDwSlotsPerSm * 148) / kcols;
  if (nchunk < 1) nchunk = 1;
  if (nchunk > (T + kDwTok - 1) / kDwTok) nchunk = (T + kDwTok - 1) / kDwTok;
  if (nchunk < 1) nchunk = 1;
  p.tchunk = ((T + nchunk - 1) / nchunk + kDwTok - 1) / kDwTok * kDwTok;
  p.nchunk = static_cast<int>((T + p.tchunk - 1) / p.tchunk);
  p.dwp = up(static_cast<size_t>(p.nchunk) * 4 * H * kMix * 4);
  p.drtc = up(pre_bwd_dr_tc_workspace_bytes(T, H));  // operands + partials of d_R with d_hc_fn
  p.dwtc = up(pre_bwd_dw_tc_workspace_bytes(T, H));  // B operand and partials of its d_hc_fn
  p.total = p.proj + p.dpt + p.brec + p.dwp + p.drtc + p.dwtc;
  return p;
}

size_t pre_backward_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0) return 0;
  return bw_plan(T, H).total;
}

int launch_pre_backward(const PreBwdArgs& a, cudaStream_t s) {
  const BwPlan plan = bw_plan(a.T, a.H);
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  float* dpt = reinterpret_cast<float*>(ws + plan.proj);
  float* brec = reinterpret_cast<float*>(ws + plan.proj + plan.dpt);
  float* dwp = reinterpret_cast<float*>(ws + plan.proj + plan.dpt + plan.brec);
  void* drtc_ws = ws + plan.proj + plan.dpt + plan.brec + plan.dwp;
  void* dwtc_ws = ws + plan.proj + plan.dpt + plan.brec + plan.dwp + plan.drtc;
  const int64_t K = 4 * a.H;
  if (a.T > 0x7fffffff) return -5;

  // 1. The projection, by the forward's kernels (its records hold raw and ss).
  PreArgs f{a.R, a.hc_fn, a.hc_scale, a.hc_base, nullptr, nullptr, nullptr, nullptr,
            a.workspace, plan.proj, a.T, a.H, a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps,
            a.post_mult};
  float* part = nullptr;
  int nrec = 0;
  const bool tc = pre_tc_supported(a.T, a.H) && aligned16(a.R) && aligned16(a.workspace) &&
                  a.T >= 128;
  // With d_y, the tensor projection also forms d_pre's sum_h d_y R_i from the tiles it streams
  // (one pass over R instead of two); H % 64 == 0 keeps each K block within one stream.
  const bool dy_fold = tc && a.dy != nullptr && a.H % 64 == 0 && aligned16(a.dy);
  int r = tc ? launch_tc_projection(f, s, &part, &nrec, dy_fold ? a.dy : nullptr)
             : launch_cc_projection(f, s, &part, &nrec);
  if (r != 0) return r;

  const bool vec = a.H % 8 == 0 && aligned16(a.R) && aligned16(a.dR) &&
                   (a.dy == nullptr || aligned16(a.dy));
  const dim3 tok(static_cast<unsigned>(a.T));
  cudaError_t e;
  // 2. d_pre (unless the projection formed it).
  if (!dy_fold) {
    e = vec ? launch_pdl(pre_bwd_dpre_kernel<true>, tok, dim3(kBwThreads), 0, s, a.dy, a.dpre,
                         a.R, dpt, a.H)
            : launch_pdl(pre_bwd_dpre_kernel<false>, tok, dim3(kBwThreads), 0, s, a.dy, a.dpre,
                         a.R, dpt, a.H);
    if (e != cudaSuccess) return -4;
  }
  // 3. Coefficients' reverse pass.
  const FinishParams fp{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};
  e = launch_pdl(pre_bwd_coef_kernel, dim3(static_cast<unsigned>((4 * a.T + 255) / 256)),
                 dim3(256), 0, s, static_cast<const float*>(part), nrec,
                 static_cast<const float*>(dpt), a.dpre, dy_fold ? 1 : 0, a.dpost, a.dcomb,
                 a.hc_scale, a.hc_base, brec,
                 a.T, K, fp);
  if (e != cudaSuccess) return -4;
  // 4. d_scale, d_base.
  e = launch_pdl(pre_bwd_param_kernel, dim3(3 + kMix), dim3(256), 0, s,
                 static_cast<const float*>(brec), a.dscale, a.dbase, a.T);
  if (e != cudaSuccess) return -4;
  // 5. d_R: on tensor cores where the shape allows, together with d_hc_fn (1: not this shape,
  // nothing launched), else column slices x token chunks on CUDA cores, one wave of
  // kDxSlotsPerSm CTAs per SM.
  int dr = 1;
  if (vec) {
    dr = launch_pre_bwd_dr_tc(a.R, a.dy, a.hc_fn, static_cast<const float*>(brec), kBrec, a.dR,
                              a.dW, drtc_ws, a.T, a.H, s);
    if (dr < 0) return dr;
  }
  if (dr == 0) {
    e = cudaSuccess;
  } else if (vec) {
    if (!ensure_smem_limit(reinterpret_cast<const void*>(pre_bwd_dx_kernel), kDxSmem)) return -4;
    const int64_t xcols = (K + kDxCols - 1) / kDxCols;
    int64_t xch = (kDxSlotsPerSm * static_cast<int64_t>(device_sm_count())) / xcols;
    if (xch < 1) xch = 1;
    if (xch > (a.T + kDxTok - 1) / kDxTok) xch = (a.T + kDxTok - 1) / kDxTok;
    const int64_t xtchunk = ((a.T + xch - 1) / xch + kDxTok - 1) / kDxTok * kDxTok;
    const dim3 g(static_cast<unsigned>(xcols),
                 static_cast<unsigned>((a.T + xtchunk - 1) / xtchunk));
    e = launch_pdl(pre_bwd_dx_kernel, g, dim3(kDxThreads), static_cast<size_t>(kDxSmem), s, a.R,
                   a.dy, a.hc_fn, static_cast<const float*>(brec), a.dR, a.T, a.H, xtchunk);
  } else {
    int64_t nb = (a.T * K + 255) / 256;
    if (nb > 148 * 16) nb = 148 * 16;
    e = launch_pdl(pre_bwd_dx_scalar_kernel, dim3(static_cast<unsigned>(nb)), dim3(256), 0, s,
                   a.R, a.dy, a.hc_fn, static_cast<const float*>(brec), a.dR, a.T, a.H);
  }
  if (e != cudaSuccess) return -4;
  // 6. d_hc_fn (unless step 5 formed it): on tensor cores where 4H % 128 == 0 (1: not this
  // shape, nothing launched), else CUDA-core partials over token chunks; then the partials'
  // in-order sum.
  int dwr = 0;
  if (dr != 0) {
    dwr = launch_pre_bwd_dw_tc(a.R, static_cast<const float*>(brec), kBrec, a.dW, dwtc_ws, a.T,
                               a.H, s);
    if (dwr < 0) return dwr;
  }
  if (dwr == 1) {
    const dim3 gw(static_cast<unsigned>((K + kDwCols - 1) / kDwCols),
                  static_cast<unsigned>(plan.nchunk));
    const bool dwvec = a.H % 8 == 0 && aligned16(a.R);
    e = dwvec ? launch_pdl(pre_bwd_dw_kernel<true>, gw, dim3(kDwThreads), 0, s, a.R,
                           static_cast<const float*>(brec), dwp, a.T, a.H, plan.tchunk)
              : launch_pdl(pre_bwd_dw_kernel<false>, gw, dim3(kDwThreads), 0, s, a.R,
                           static_cast<const float*>(brec), dwp, a.T, a.H, plan.tchunk);
    if (e != cudaSuccess) return -4;
    int64_t nb = (K * kMix + 255) / 256;
    if (nb > 148 * 8) nb = 148 * 8;
    e = launch_pdl(pre_bwd_dw_sum_kernel, dim3(static_cast<unsigned>(nb)), dim3(256), 0, s,
                   static_cast<const float*>(dwp), a.dW, K * kMix, plan.nchunk);
    if (e != cudaSuccess) return -4;
    note_launches(2);
  }
  // [dpre], coef, param, [d_R on CUDA cores] (the tensor-core forms count their own launches).
  note_launches((dy_fold ? 2 : 3) + (dr == 0 ? 0 : 1));
  return 0;
}

}  // namespace mhc
