// Standalone Sinkhorn normalisation of [T][4][4] logits ("FlashInfer mHC module deep dive" §3.4,
// §5.2: row softmax with row-max shift, eps added to every entry, then rounds of row and column
// normalisation by plain sums).
//
// Two forms with identical results: four lanes per token, lane q owning row q (16 bytes in, 16 bytes
// out; column sums across the quad with xor shuffles), which keeps many threads busy for a few
// thousand tokens; and one thread per token (the whole block in 16 registers, no shuffles, half the
// instructions per token), for calls with many tokens, where the rounds' arithmetic is the bound.
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

template <bool kAligned>
__global__ void __launch_bounds__(256) sinkhorn_kernel(const float* logits, float* comb, int64_t T,
                                                       int iters, float eps) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t gid = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  const int64_t t = gid >> 2;
  const int q = static_cast<int>(gid & 3);
  const bool live = t < T;
  float a[4] = {0.f, 0.f, 0.f, 0.f};
  if (live) {
    const float* src = logits + t * 16 + q * 4;
    if (kAligned) {
      const float4 v = *reinterpret_cast<const float4*>(src);
      a[0] = v.x, a[1] = v.y, a[2] = v.z, a[3] = v.w;
    } else {
#pragma unroll
      for (int n = 0; n < 4; ++n) a[n] = src[n];
    }
  }
  sinkhorn_quad(a, iters, eps);  // every lane of the warp takes part
  if (live) {
    float* dst = comb + t * 16 + q * 4;
    if (kAligned) {
      *reinterpret_cast<float4*>(dst) = make_float4(a[0], a[1], a[2], a[3]);
    } else {
#pragma unroll
      for (int n = 0; n < 4; ++n) dst[n] = a[n];
    }
  }
}

template <bool kAligned>
__global__ void __launch_bounds__(256) sinkhorn_thread_kernel(const float* logits, float* comb,
                                                              int64_t T, int iters, float eps) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t t = blockIdx.x * (int64_t)blockDim.x + threadIdx.x;
  if (t >= T) return;
  float a[16];
  const float* src = logits + t * 16;
  if (kAligned) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float4 v = *reinterpret_cast<const float4*>(src + 4 * q);
      a[4 * q] = v.x, a[4 * q + 1] = v.y, a[4 * q + 2] = v.z, a[4 * q + 3] = v.w;
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) a[i] = src[i];
  }
  sinkhorn_thread(a, iters, eps);
  float* dst = comb + t * 16;
  if (kAligned) {
#pragma unroll
    for (int q = 0; q < 4; ++q)
      *reinterpret_cast<float4*>(dst + 4 * q) =
          make_float4(a[4 * q], a[4 * q + 1], a[4 * q + 2], a[4 * q + 3]);
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) dst[i] = a[i];
  }
}

// Tokens from which the one-thread-per-token form fills the GPU (256 CTAs of 256 threads).
constexpr int64_t kSkThreadMinTokens = 65536;

int launch_sinkhorn(const float* logits, float* comb, int64_t T, int iters, float eps,
                    cudaStream_t s) {
  const int threads = 256;
  const bool al = aligned16(logits) && aligned16(comb);
  if (T >= kSkThreadMinTokens) {
    const int64_t blocks = (T + threads - 1) / threads;
    if (blocks > 0x7fffffff) return -1;
    const dim3 grid(static_cast<unsigned>(blocks));
    const cudaError_t e =
        al ? launch_pdl(sinkhorn_thread_kernel<true>, grid, dim3(threads), 0, s, logits, comb, T,
                        iters, eps)
           : launch_pdl(sinkhorn_thread_kernel<false>, grid, dim3(threads), 0, s, logits, comb, T,
                        iters, eps);
    note_launches(1);
    return e == cudaSuccess ? 0 : -4;
  }
  const int64_t blocks = (4 * T + threads - 1) / threads;
  if (blocks > 0x7fffffff) return -1;
  const dim3 grid(static_cast<unsigned>(blocks));
  const cudaError_t e =
      al ? launch_pdl(sinkhorn_kernel<true>, grid, dim3(threads), 0, s, logits, comb, T, iters, eps)
          : launch_pdl(sinkhorn_kernel<false>, grid, dim3(threads), 0, s, logits, comb, T, iters,
                       eps);
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

}  // namespace mhc
