// mHC post-map: out[t][n][h] = bf16_rn(x[t][h]*post[t][n] + sum_o R[t][o][h]*comb[t][o][n]).
// "FlashInfer mHC module deep dive" §2.1 (formula) and §2.3 (vec8 / persistent / scalar paths);
// glm5next_mhc.rs glm_hc_post (out may alias the residual).
//
// Every kernel reads the four streams of an element before it writes that element, and each
// element is owned by one thread (or one staged tile), so out == R is safe.
//
// Arithmetic per output, in fp32: acc = x*post[n]; acc = fma(R[o], comb[o][n], acc) for o = 0..3;
// round to bf16 (nearest even).
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

struct Coef20 {
  float4 post;  // post[0..3]
  float4 c[4];  // c[o] = comb[o][0..3]
};

template <bool kAlignedCoef>
__device__ __forceinline__ Coef20 load_coef(const float* post, const float* comb, int64_t t) {
  Coef20 k;
  if (kAlignedCoef) {
    k.post = __ldg(reinterpret_cast<const float4*>(post + t * 4));
#pragma unroll
    for (int o = 0; o < 4; ++o) k.c[o] = __ldg(reinterpret_cast<const float4*>(comb + t * 16 + o * 4));
  } else {
    const float* p = post + t * 4;
    k.post = make_float4(__ldg(p), __ldg(p + 1), __ldg(p + 2), __ldg(p + 3));
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      const float* q = comb + t * 16 + o * 4;
      k.c[o] = make_float4(__ldg(q), __ldg(q + 1), __ldg(q + 2), __ldg(q + 3));
    }
  }
  return k;
}

__device__ __forceinline__ float mix1(float x, float p, float r0, float r1, float r2, float r3,
                                      float c0, float c1, float c2, float c3) {
  float acc = x * p;
  acc = fmaf(r0, c0, acc);
  acc = fmaf(r1, c1, acc);
  acc = fmaf(r2, c2, acc);
  acc = fmaf(r3, c3, acc);
  return acc;
}

// Two packed bf16 lanes (element pair) of all four output streams.
__device__ __forceinline__ void mix_pair(uint32_t xv, uint32_t r0, uint32_t r1, uint32_t r2,
                                         uint32_t r3, const Coef20& k, uint32_t (&o)[4]) {
  const float xl = bf16_lo(xv), xh = bf16_hi(xv);
  const float a0 = bf16_lo(r0), a1 = bf16_lo(r1), a2 = bf16_lo(r2), a3 = bf16_lo(r3);
  const float b0 = bf16_hi(r0), b1 = bf16_hi(r1), b2 = bf16_hi(r2), b3 = bf16_hi(r3);
  o[0] = pack_bf16x2(mix1(xl, k.post.x, a0, a1, a2, a3, k.c[0].x, k.c[1].x, k.c[2].x, k.c[3].x),
                     mix1(xh, k.post.x, b0, b1, b2, b3, k.c[0].x, k.c[1].x, k.c[2].x, k.c[3].x));
  o[1] = pack_bf16x2(mix1(xl, k.post.y, a0, a1, a2, a3, k.c[0].y, k.c[1].y, k.c[2].y, k.c[3].y),
                     mix1(xh, k.post.y, b0, b1, b2, b3, k.c[0].y, k.c[1].y, k.c[2].y, k.c[3].y));
  o[2] = pack_bf16x2(mix1(xl, k.post.z, a0, a1, a2, a3, k.c[0].z, k.c[1].z, k.c[2].z, k.c[3].z),
                     mix1(xh, k.post.z, b0, b1, b2, b3, k.c[0].z, k.c[1].z, k.c[2].z, k.c[3].z));
  o[3] = pack_bf16x2(mix1(xl, k.post.w, a0, a1, a2, a3, k.c[0].w, k.c[1].w, k.c[2].w, k.c[3].w),
                     mix1(xh, k.post.w, b0, b1, b2, b3, k.c[0].w, k.c[1].w, k.c[2].w, k.c[3].w));
}

// 8 consecutive elements (one 16-byte vector per stream).
__device__ __forceinline__ void mix_vec8(const uint4& xv, const uint4 (&r)[4], const Coef20& k,
                                         uint4 (&out)[4]) {
  uint32_t o[4];
  mix_pair(xv.x, r[0].x, r[1].x, r[2].x, r[3].x, k, o);
  out[0].x = o[0], out[1].x = o[1], out[2].x = o[2], out[3].x = o[3];
  mix_pair(xv.y, r[0].y, r[1].y, r[2].y, r[3].y, k, o);
  out[0].y = o[0], out[1].y = o[1], out[2].y = o[2], out[3].y = o[3];
  mix_pair(xv.z, r[0].z, r[1].z, r[2].z, r[3].z, k, o);
  out[0].z = o[0], out[1].z = o[1], out[2].z = o[2], out[3].z = o[3];
  mix_pair(xv.w, r[0].w, r[1].w, r[2].w, r[3].w, k, o);
  out[0].w = o[0], out[1].w = o[1], out[2].w = o[2], out[3].w = o[3];
}

// ------------------------------------------------------------------------------ vec8 kernel
// One thread per (token, 8-element group), flattened as u = t*H8 + v. kInPlace selects the
// coherent load path (out aliases R).
template <bool kInPlace>
__global__ void __launch_bounds__(256) post_vec8_kernel(const uint16_t* __restrict__ x,
                                                        const uint16_t* R,
                                                        const float* __restrict__ post,
                                                        const float* __restrict__ comb,
                                                        uint16_t* out, int64_t T, int64_t H8) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t total = T * H8;
  const int64_t H = H8 * 8;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = u / H8;
    const int64_t v = u - t * H8;
    const uint16_t* rrow = R + t * 4 * H + v * 8;
    const uint4 xv = ld_stream_ro(x + t * H + v * 8);
    uint4 r[4];
#pragma unroll
    for (int o = 0; o < 4; ++o) r[o] = kInPlace ? ld_stream(rrow + o * H) : ld_stream_ro(rrow + o * H);
    const Coef20 k = load_coef<true>(post, comb, t);
    uint4 res[4];
    mix_vec8(xv, r, k, res);
    uint16_t* orow = out + t * 4 * H + v * 8;
#pragma unroll
    for (int n = 0; n < 4; ++n) st_stream(orow + n * H, res[n]);
  }
}

// ------------------------------------------------------------------------------ scalar kernel
// One thread per (token, element). Any H, any alignment.
template <bool kAlignedCoef>
__global__ void __launch_bounds__(256) post_scalar_kernel(const uint16_t* x, const uint16_t* R,
                                                          const float* post, const float* comb,
                                                          uint16_t* out, int64_t T, int64_t H) {
  pdl_wait();  // launched as a programmatic dependent of the previous grid
  pdl_trigger();
  const int64_t total = T * H;
  for (int64_t e = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; e < total;
       e += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = e / H;
    const int64_t h = e - t * H;
    const uint16_t* rr = R + t * 4 * H + h;
    const float xv = bf16_to_f32(x[t * H + h]);
    const float r0 = bf16_to_f32(rr[0]), r1 = bf16_to_f32(rr[H]), r2 = bf16_to_f32(rr[2 * H]),
                r3 = bf16_to_f32(rr[3 * H]);
    const Coef20 k = load_coef<kAlignedCoef>(post, comb, t);
    uint16_t* oo = out + t * 4 * H + h;
    oo[0] = f32_to_bf16(mix1(xv, k.post.x, r0, r1, r2, r3, k.c[0].x, k.c[1].x, k.c[2].x, k.c[3].x));
    oo[H] = f32_to_bf16(mix1(xv, k.post.y, r0, r1, r2, r3, k.c[0].y, k.c[1].y, k.c[2].y, k.c[3].y));
    oo[2 * H] =
        f32_to_bf16(mix1(xv, k.post.z, r0, r1, r2, r3, k.c[0].z, k.c[1].z, k.c[2].z, k.c[3].z));
    oo[3 * H] =
        f32_to_bf16(mix1(xv, k.post.w, r0, r1, r2, r3, k.c[0].w, k.c[1].w, k.c[2].w, k.c[3].w));
  }
}

// ------------------------------------------------------------------------------ persistent kernel
// Persistent grid; each CTA walks tiles (token t, chunk c of kChunk elements) with a stride of
// gridDim.x. One producer thread stages the five input rows of a tile (x and R[0..3]) into a
// shared-memory ring with 1-D bulk copies completing on an mbarrier; kConsumers threads compute
// 8 elements each from shared memory and store straight to global. Empty barriers return a stage
// to the producer. All waits are bounded.
constexpr int kPostChunk = 1024;                       // elements per row chunk
constexpr int kPostStages = 6;
constexpr int kPostConsumers = kPostChunk / 8;         // 128 threads, 8 elements each
constexpr int kPostThreads = kPostConsumers + 32;      // + one producer warp
constexpr int kPostStageBytes = 5 * kPostChunk * 2;    // 10 KB
constexpr int kPostSmem = kPostStages * kPostStageBytes + 2 * kPostStages * 8;

__global__ void __launch_bounds__(kPostThreads) post_persistent_kernel(
    const uint16_t* __restrict__ x, const uint16_t* R, const float* __restrict__ post,
    const float* __restrict__ comb, uint16_t* out, int64_t T, int64_t H) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint16_t* stage_base = reinterpret_cast<uint16_t*>(smem);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kPostStages * kPostStageBytes);
  uint64_t* empty = full + kPostStages;

  const int64_t chunks = (H + kPostChunk - 1) / kPostChunk;
  const int64_t tiles = T * chunks;
  const int tid = threadIdx.x;

  if (tid == 0) {
    for (int s = 0; s < kPostStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kPostConsumers);
    }
    fence_mbarrier_init();
  }
  __syncthreads();
  pdl_wait();  // launched as a programmatic dependent of the previous grid in the stream
  pdl_trigger();

  if (tid >= kPostConsumers) {
    // Producer warp: lane 0 issues the copies.
    if (tid == kPostConsumers) {
      int s = 0;
      uint32_t phase = 0;
      int issued = 0;
      bool ok = true;
      for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
        if (issued >= kPostStages && !mbar_wait(&empty[s], phase ^ 1u, 1)) {
          ok = false;
          break;
        }
        const int64_t t = tile / chunks;
        const int64_t c = tile - t * chunks;
        const int64_t h0 = c * kPostChunk;
        const uint32_t n = static_cast<uint32_t>((H - h0 < kPostChunk ? H - h0 : static_cast<int64_t>(kPostChunk)));
        const uint32_t bytes = n * 2u;
        uint16_t* st = stage_base + s * (5 * kPostChunk);
        mbar_arrive_expect_tx(&full[s], 5u * bytes);
        bulk_g2s(st, x + t * H + h0, bytes, &full[s]);
#pragma unroll
        for (int o = 0; o < 4; ++o)
          bulk_g2s(st + (o + 1) * kPostChunk, R + (t * 4 + o) * H + h0, bytes, &full[s]);
        ++issued;
        if (++s == kPostStages) { s = 0; phase ^= 1u; }
      }
      // Drain: do not leave the CTA while copies into its shared memory are in flight. Stage i was
      // filled n_i times; its last fill completes the phase with parity (n_i - 1) & 1.
      if (!ok) {
        for (int i = 0; i < kPostStages; ++i) {
          const int n_i = issued / kPostStages + (i < issued % kPostStages ? 1 : 0);
          if (n_i > 0) mbar_wait(&full[i], static_cast<uint32_t>((n_i - 1) & 1), 2);
        }
      }
    }
    return;
  }

  // Consumers.
  int s = 0;
  uint32_t phase = 0;
  for (int64_t tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    if (!mbar_wait(&full[s], phase, 3)) return;
    const int64_t t = tile / chunks;
    const int64_t c = tile - t * chunks;
    const int64_t h0 = c * kPostChunk;
    const int64_t n = (H - h0 < kPostChunk ? H - h0 : static_cast<int64_t>(kPostChunk));
    const uint16_t* st = stage_base + s * (5 * kPostChunk);
    const int e = tid * 8;
    if (e < n) {
      const uint4 xv = *reinterpret_cast<const uint4*>(st + e);
      uint4 r[4];
#pragma unroll
      for (int o = 0; o < 4; ++o) r[o] = *reinterpret_cast<const uint4*>(st + (o + 1) * kPostChunk + e);
      const Coef20 k = load_coef<true>(post, comb, t);
      uint4 res[4];
      mix_vec8(xv, r, k, res);
      uint16_t* orow = out + t * 4 * H + h0 + e;
#pragma unroll
      for (int q = 0; q < 4; ++q) st_stream(orow + q * H, res[q]);
    }
    mbar_arrive(&empty[s]);
    if (++s == kPostStages) { s = 0; phase ^= 1u; }
  }
}

// ------------------------------------------------------------------------------ launchers

static int grid_for(int64_t work, int threads, int max_blocks) {
  int64_t b = (work + threads - 1) / threads;
  if (b > max_blocks) b = max_blocks;
  if (b < 1) b = 1;
  return static_cast<int>(b);
}

int launch_post_vec8(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                     uint16_t* out, int64_t T, int64_t H, cudaStream_t s) {
  const int64_t H8 = H / 8;
  const int threads = 256;
  const int blocks = grid_for(T * H8, threads, device_sm_count() * 64);
  cudaError_t e;
  if (out == R)
    e = launch_pdl(post_vec8_kernel<true>, dim3(blocks), dim3(threads), 0, s, x, R,
                   post, comb, out, T, H8);
  else
    e = launch_pdl(post_vec8_kernel<false>, dim3(blocks), dim3(threads), 0, s, x, R,
                   post, comb, out, T, H8);
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

int launch_post_scalar(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                       uint16_t* out, int64_t T, int64_t H, cudaStream_t s) {
  const int threads = 256;
  const int blocks = grid_for(T * H, threads, device_sm_count() * 64);
  const bool aligned = aligned16(post) && aligned16(comb);
  cudaError_t e;
  if (aligned)
    e = launch_pdl(post_scalar_kernel<true>, dim3(blocks), dim3(threads), 0, s, x, R,
                   post, comb, out, T, H);
  else
    e = launch_pdl(post_scalar_kernel<false>, dim3(blocks), dim3(threads), 0, s, x, R,
                   post, comb, out, T, H);
  note_launches(1);
  return e == cudaSuccess ? 0 : -4;
}

int launch_post_persistent(const uint16_t* x, const uint16_t* R, const float* post,
                           const float* comb, uint16_t* out, int64_t T, int64_t H,
                           cudaStream_t s) {
  if (!ensure_smem_limit(reinterpret_cast<const void*>(post_persistent_kernel), kPostSmem)) return -4;
  const int64_t tiles = T * ((H + kPostChunk - 1) / kPostChunk);
  int64_t blocks = static_cast<int64_t>(device_sm_count()) * 3;  // 3 x 61 KB of stages per SM
  if (blocks > tiles) blocks = tiles;
  if (launch_pdl(post_persistent_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kPostThreads),
                 static_cast<size_t>(kPostSmem), s, x, R, post, comb, out, T, H) != cudaSuccess)
    return -4;
  note_launches(1);
  return 0;
}

}  // namespace mhc
