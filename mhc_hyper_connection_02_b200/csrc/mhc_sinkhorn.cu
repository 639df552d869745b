// Standalone Sinkhorn normalisation of [T][4][4] logits ("FlashInfer mHC module deep dive" §3.4,
// §5.2: row softmax with row-max shift, eps added to every entry, then rounds of row and column
// normalisation by plain sums).
//
// Four lanes per token, lane q owning row q (16 bytes in, 16 bytes out): rows normalise in
// registers, column sums reduce across the quad with xor shuffles.
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

int launch_sinkhorn(const float* logits, float* comb, int64_t T, int iters, float eps,
                    cudaStream_t s) {
  const int threads = 256;
  const int64_t blocks = (4 * T + threads - 1) / threads;
  if (blocks > 0x7fffffff) return -1;
  const dim3 grid(static_cast<unsigned>(blocks));
  const cudaError_t e =
      (aligned16(logits) && aligned16(comb))
          ? launch_pdl(sinkhorn_kernel<true>, grid, dim3(threads), 0, s, logits, comb, T, iters, eps)
          : launch_pdl(sinkhorn_kernel<false>, grid, dim3(threads), 0, s, logits, comb, T, iters,
                       eps);
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

}  // namespace mhc
