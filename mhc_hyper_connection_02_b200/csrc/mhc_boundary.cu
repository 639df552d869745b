// The model-boundary operations either side of the layer stack: expand (first layer: the hidden row
// becomes every stream) and head (last layer: the streams collapse to one row).
//
// glm5next_mhc.rs glm_hc_expand ("broadcast each hidden row into its hc_mult highway streams") and
// hc_head_mean ("the unweighted mean of the hc_mult streams"); hyper_connection_dispatch.rs
// hc_head_site (the weighted head takes hc_fn / hc_scale / hc_base, a norm eps and hc_eps; its
// kernel is not shown). The weighted head is formed by the pre-map's machinery on a projection
// padded from 4 to 24 columns (see mhc_api.cu); this file holds its padding kernel.
//
// Streams here are the library's bf16 [T][4][H] residual (GLM keeps fp32 streams).
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

// streams[t][i][:] = hidden[t][:] for i < 4; one thread per 8 columns (16-byte accesses).
__global__ void __launch_bounds__(256) expand_vec8_kernel(const uint16_t* __restrict__ hidden,
                                                          uint16_t* __restrict__ streams,
                                                          int64_t T, int64_t H8) {
  const int64_t total = T * H8;
  const int64_t H = H8 * 8;
  pdl_wait();
  pdl_trigger();
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = u / H8;
    const int64_t v = u - t * H8;
    const uint4 x = ld_stream_ro(hidden + t * H + v * 8);
    uint16_t* o = streams + t * 4 * H + v * 8;
#pragma unroll
    for (int i = 0; i < 4; ++i) st_plain(o + i * H, x);
  }
}

__global__ void __launch_bounds__(256) expand_scalar_kernel(const uint16_t* __restrict__ hidden,
                                                            uint16_t* __restrict__ streams,
                                                            int64_t T, int64_t H) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t total = T * H;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = u / H;
    const int64_t h = u - t * H;
    const uint16_t x = hidden[u];
#pragma unroll
    for (int i = 0; i < 4; ++i) streams[(t * 4 + i) * H + h] = x;
  }
}

// y[t][h] = bf16_rn(((R0 + R1) + R2 + R3) * 0.25), fp32 sums (the scaling by 1/4 is exact).
__global__ void __launch_bounds__(256) head_mean_vec8_kernel(const uint16_t* __restrict__ R,
                                                             uint16_t* __restrict__ y, int64_t T,
                                                             int64_t H8) {
  const int64_t total = T * H8;
  const int64_t H = H8 * 8;
  pdl_wait();
  pdl_trigger();
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = u / H8;
    const int64_t v = u - t * H8;
    const uint16_t* rr = R + t * 4 * H + v * 8;
    uint4 rv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) rv[i] = ld_stream_ro(rr + i * H);
    uint32_t o[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const uint32_t w0 = (&rv[0].x)[q], w1 = (&rv[1].x)[q], w2 = (&rv[2].x)[q],
                     w3 = (&rv[3].x)[q];
      const float lo = (((bf16_lo(w0) + bf16_lo(w1)) + bf16_lo(w2)) + bf16_lo(w3)) * 0.25f;
      const float hi = (((bf16_hi(w0) + bf16_hi(w1)) + bf16_hi(w2)) + bf16_hi(w3)) * 0.25f;
      o[q] = pack_bf16x2(lo, hi);
    }
    st_plain(y + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

__global__ void __launch_bounds__(256) head_mean_scalar_kernel(const uint16_t* __restrict__ R,
                                                               uint16_t* __restrict__ y, int64_t T,
                                                               int64_t H) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t total = T * H;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t t = u / H;
    const int64_t h = u - t * H;
    const uint16_t* rr = R + t * 4 * H + h;
    const float s = ((bf16_to_f32(rr[0]) + bf16_to_f32(rr[H])) + bf16_to_f32(rr[2 * H])) +
                    bf16_to_f32(rr[3 * H]);
    y[u] = f32_to_bf16(s * 0.25f);
  }
}

// Weighted head: hc_fn [K][4] -> fn24 [K][24] (columns 4..23 zero); scale3 = (scale[0], 1, 1),
// base24 = (base[0..3], 0, ...).
__global__ void __launch_bounds__(256) head_pad_kernel(const float* __restrict__ fn4,
                                                       const float* __restrict__ scale1,
                                                       const float* __restrict__ base4,
                                                       float* __restrict__ fn24,
                                                       float* __restrict__ sb, int64_t K) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t total = K * kMix;
  for (int64_t u = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; u < total;
       u += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int64_t k = u / kMix;
    const int j = static_cast<int>(u - k * kMix);
    fn24[u] = j < 4 ? fn4[k * 4 + j] : 0.0f;
  }
  if (blockIdx.x == 0 && threadIdx.x < 3 + kMix) {
    const int i = threadIdx.x;
    float v;
    if (i < 3)
      v = i == 0 ? scale1[0] : 1.0f;
    else
      v = i - 3 < 4 ? base4[i - 3] : 0.0f;
    sb[i] = v;
  }
}

static unsigned stream_grid(int64_t units) {
  int64_t b = (units + 255) / 256;
  const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
  if (b > cap) b = cap;
  return static_cast<unsigned>(b < 1 ? 1 : b);
}

int launch_expand(const uint16_t* hidden, uint16_t* streams, int64_t T, int64_t H,
                  cudaStream_t s) {
  cudaError_t e;
  if (H % 8 == 0 && aligned16(hidden) && aligned16(streams)) {
    e = launch_pdl(expand_vec8_kernel, dim3(stream_grid(T * (H / 8))), dim3(256), 0, s, hidden,
                   streams, T, H / 8);
  } else {
    e = launch_pdl(expand_scalar_kernel, dim3(stream_grid(T * H)), dim3(256), 0, s, hidden, streams,
                   T, H);
  }
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

int launch_head_mean(const uint16_t* R, uint16_t* y, int64_t T, int64_t H, cudaStream_t s) {
  cudaError_t e;
  if (H % 8 == 0 && aligned16(R) && aligned16(y)) {
    e = launch_pdl(head_mean_vec8_kernel, dim3(stream_grid(T * (H / 8))), dim3(256), 0, s, R, y,
                   T, H / 8);
  } else {
    e = launch_pdl(head_mean_scalar_kernel, dim3(stream_grid(T * H)), dim3(256), 0, s, R, y, T, H);
  }
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

int launch_head_pad(const float* fn4, const float* scale1, const float* base4, float* fn24,
                    float* sb, int64_t H, cudaStream_t s) {
  const int64_t K = 4 * H;
  const cudaError_t e = launch_pdl(head_pad_kernel, dim3(stream_grid(K * kMix)), dim3(256), 0, s,
                                   fn4, scale1, base4, fn24, sb, K);
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

}  // namespace mhc
