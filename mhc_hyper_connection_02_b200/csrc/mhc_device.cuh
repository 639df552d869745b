// Device-side helpers shared by the mHC kernels (sm_100a): bf16 packing, 16-byte global
// loads/stores with cache hints, mbarrier and bulk-copy wrappers with bounded waits, and the
// per-token coefficient math (gates and the 4x4 Sinkhorn).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace mhc {

constexpr int kHC = 4;
constexpr int kMix = 24;

// Status word that bounded waits set when they give up; read and cleared by mhc_device_status().
// Defined here: the library is a single translation unit (libmhc.cu).
__device__ int g_device_status = 0;

// Bounded waits give up after this many nanoseconds of %globaltimer.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

__device__ __forceinline__ unsigned long long global_timer_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void report_timeout(int where) {
  atomicCAS(&g_device_status, 0, -6 /* MHC_ERR_TIMEOUT */);
  (void)where;
}

// ------------------------------------------------------------------------------ dependent launch

// Programmatic dependent launch. pdl_wait blocks until every grid this one depends on in the stream
// has completed and its memory operations are visible (it returns at once for a grid launched
// without the programmatic-serialisation attribute); every thread calls it before its first access
// to global memory. pdl_trigger lets the next grid in the stream start launching once all CTAs of
// this one have triggered or exited; that grid still waits in its own pdl_wait.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ------------------------------------------------------------------------------ bf16 packing

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }
__device__ __forceinline__ float bf16_to_f32(uint16_t v) {
  return __uint_as_float(static_cast<uint32_t>(v) << 16);
}

// Round two floats to bf16 (nearest even) and pack them, `a` in the low half.
__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
__device__ __forceinline__ uint16_t f32_to_bf16(float a) {
  __nv_bfloat16 v = __float2bfloat16_rn(a);
  return *reinterpret_cast<uint16_t*>(&v);
}

// ------------------------------------------------------------------------------ 16-byte memory ops

// Streaming read-only load (data not written by this kernel): non-coherent path, no L1 allocation.
__device__ __forceinline__ uint4 ld_stream_ro(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}
// Streaming load of data this kernel may later overwrite (in-place): coherent path.
__device__ __forceinline__ uint4 ld_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p)
               : "memory");
  return v;
}
__device__ __forceinline__ void st_stream(void* p, uint4 v) {
  asm volatile("st.global.cs.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}
__device__ __forceinline__ void st_plain(void* p, uint4 v) {
  asm volatile("st.global.v4.u32 [%0], {%1,%2,%3,%4};" ::"l"(p), "r"(v.x), "r"(v.y), "r"(v.z),
               "r"(v.w)
               : "memory");
}

// ------------------------------------------------------------------------------ mbarrier + bulk copy

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}
__device__ __forceinline__ void fence_mbarrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(smem_u32(bar))
      : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(
          smem_u32(bar)),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Wait for the phase with the given parity to complete. Returns false (and records a timeout) if
// it has not completed within limit_ns; the caller then stops using the pipeline. Also returns
// false once another wait has recorded a timeout.
__device__ __forceinline__ bool mbar_wait_for(uint64_t* bar, uint32_t parity, int where,
                                              unsigned long long limit_ns) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((i & 255u) == 0) {
      if (*reinterpret_cast<volatile int*>(&g_device_status) != 0) return false;
      if (global_timer_ns() - t0 > limit_ns) {
        report_timeout(where);
        return false;
      }
    }
  }
}
// The kernels' waits use the library-wide limit.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, int where) {
  return mbar_wait_for(bar, parity, where, kWaitLimitNs);
}

// 1-D bulk copy global -> shared (TMA engine), completion counted on `bar` in bytes. Both
// addresses 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(void* smem_dst, const void* gmem_src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
          smem_u32(smem_dst)),
      "l"(gmem_src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Named barrier over `nthreads` threads that also ORs a predicate: every participant gets the same
// answer, so a decision taken on it (such as stopping after a timeout) keeps the barrier sequence
// matched.
__device__ __forceinline__ bool named_bar_or(int id, int nthreads, bool pred) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\tsetp.ne.u32 p, %1, 0;\n\t"
      "bar.red.or.pred q, %2, %3, p;\n\tselp.u32 %0, 1, 0, q;\n\t}"
      : "=r"(r)
      : "r"(pred ? 1u : 0u), "r"(id), "r"(nthreads)
      : "memory");
  return r != 0;
}

// ------------------------------------------------------------------------------ cross-CTA counters

// Acquire load at gpu scope: later reads of this thread see what the releasing writers published.
__device__ __forceinline__ int ld_acquire_gpu(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Everything this thread has observed (including, through a CTA-scope barrier before it, other
// threads' stores) is visible at gpu scope before the add.
__device__ __forceinline__ void red_release_add_gpu(int* p, int v) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v)
               : "memory");
}

// ------------------------------------------------------------------------------ coefficient math

__device__ __forceinline__ float sigmoidf_ieee(float v) { return 1.0f / (1.0f + expf(-v)); }

// 1/s for a positive normal s: the hardware approximate reciprocal refined by one Newton-Raphson
// step r1 = r0 + r0 * (1 - s * r0) (the textbook iteration for 1/s, e.g. Muller et al.,
// "Handbook of Floating-Point Arithmetic", ch. 5), which roughly doubles the correct bits of r0;
// the result is within about an ulp of the correctly rounded reciprocal.
__device__ __forceinline__ float recip_nr(float s) {
  float r0;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(r0) : "f"(s));
  const float e = fmaf(-s, r0, 1.0f);
  return fmaf(r0, e, r0);
}

// Sinkhorn on one 4x4 block held as 4 rows by 4 cooperating lanes: lane q (= lane & 3 within its
// quad) owns row q. The row goes through a softmax (row maximum subtracted first) and eps is added
// to every entry; then `iters` rounds of (row /= rowsum, column /= colsum) with plain sums
// ("FlashInfer mHC module deep dive" §5.2 test reference, §3.4 phase 2). Every division is a
// multiplication by recip_nr of the sum. Column sums reduce across the quad with xor shuffles.
// All 32 lanes of the warp must call it (inactive quads pass any finite values).
__device__ __forceinline__ void sinkhorn_quad(float (&a)[4], int iters, float eps) {
  // Callers reach here from lane-dependent branches; reconverge once so that the loop's
  // full-warp shuffles run with the whole warp together (measured: a diverged entry made each
  // round about ten times slower).
  __syncwarp();
  const float m = fmaxf(fmaxf(a[0], a[1]), fmaxf(a[2], a[3]));
#pragma unroll
  for (int n = 0; n < 4; ++n) a[n] = expf(a[n] - m);
  const float rs0 = recip_nr(((a[0] + a[1]) + a[2]) + a[3]);
#pragma unroll
  for (int n = 0; n < 4; ++n) a[n] = fmaf(a[n], rs0, eps);
  for (int it = 0; it < iters; ++it) {
    const float rr = recip_nr(((a[0] + a[1]) + a[2]) + a[3]);
#pragma unroll
    for (int n = 0; n < 4; ++n) a[n] *= rr;
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      float c = a[n] + __shfl_xor_sync(0xffffffffu, a[n], 1);
      c = c + __shfl_xor_sync(0xffffffffu, c, 2);
      a[n] *= recip_nr(c);
    }
  }
}

// The same Sinkhorn for one whole 4x4 block in one thread (a[4 * o + n], [old][new]): no
// shuffles, half the instructions per token of the lane-quad form, for calls with many tokens.
// Sums are associated exactly as in sinkhorn_quad (rows ((a0 + a1) + a2) + a3, columns
// (a0 + a1) + (a2 + a3)), so the two forms give identical results.
__device__ __forceinline__ void sinkhorn_thread(float (&a)[16], int iters, float eps) {
#pragma unroll
  for (int o = 0; o < 4; ++o) {
    float* r = a + 4 * o;
    const float m = fmaxf(fmaxf(r[0], r[1]), fmaxf(r[2], r[3]));
#pragma unroll
    for (int n = 0; n < 4; ++n) r[n] = expf(r[n] - m);
    const float rs0 = recip_nr(((r[0] + r[1]) + r[2]) + r[3]);
#pragma unroll
    for (int n = 0; n < 4; ++n) r[n] = fmaf(r[n], rs0, eps);
  }
  for (int it = 0; it < iters; ++it) {
#pragma unroll
    for (int o = 0; o < 4; ++o) {
      float* r = a + 4 * o;
      const float rr = recip_nr(((r[0] + r[1]) + r[2]) + r[3]);
#pragma unroll
      for (int n = 0; n < 4; ++n) r[n] *= rr;
    }
#pragma unroll
    for (int n = 0; n < 4; ++n) {
      const float rc = recip_nr((a[n] + a[4 + n]) + (a[8 + n] + a[12 + n]));
#pragma unroll
      for (int o = 0; o < 4; ++o) a[4 * o + n] *= rc;
    }
  }
}

}  // namespace mhc
