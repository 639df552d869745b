// mHC pre-map with the projection on tcgen05 tensor cores.
//
// The projection raw[t][j] = sum_k R[t][k] * hc_fn[k][j] (k = i*H + h over the flattened [4H] row,
// j < 24) is the one dense contraction of the path ("FlashInfer mHC module deep dive" §3.4 and
// §5.2: mixes = dot_mix * rstd; glm5next_mhc.rs: hc_mix). R is bf16 and exact; hc_fn is fp32, so
// it is split exactly into three bf16 terms hi + mid + lo (each the round-to-nearest of what the
// previous ones leave: 8 + 8 + 8 significand bits cover fp32's 24) and the B operand holds the 72
// columns [hi | mid | lo] padded to N = 80. Products are exact in the fp32 accumulator; the three
// column groups are summed as (lo + mid) + hi in the epilogue.
//
// Kernels (one call):
//   split   hc_fn [4H][24] fp32 -> Bw [80][4H] bf16 (K contiguous) in the workspace.
//   proj    grid (token tiles of 128, K splits). Warp 0 issues TMA loads of R [128 x 64] and
//           Bw [80 x 64] tiles (128-byte swizzle) into a 6-stage ring; warp 1 issues
//           tcgen05.mma M=128 N=80 K=16 (four per 64-wide K block) into a TMEM accumulator;
//           warps 2-5 sum the squares of their token rows from the same shared-memory tiles and,
//           after the last block, read the accumulator (tcgen05.ld) and write the split record
//           [split][t][32] = raw[0..23], ss -- the record format of the CUDA-core path.
//   finish  the CUDA-core path's finish kernel: sums the split records in a fixed order, forms
//           rstd, the logits, gates and Sinkhorn, and aggregates y.
#include <cuda.h>

#include <mutex>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kTcM = 128;                          // tokens per tile (MMA M)
constexpr int kTcN = 80;                           // 3 x 24 split columns + 8 zero rows
constexpr int kTcKB = 64;                          // K per block: one 128-byte swizzled row
constexpr int kTcStages = 6;
constexpr int kTcABytes = kTcM * kTcKB * 2;        // 16384
constexpr int kTcBBytes = kTcN * kTcKB * 2;        // 10240
constexpr int kTcStageBytes = kTcABytes + kTcBBytes;  // 26624 = 26 x 1024
constexpr int kTcThreads = 192;
constexpr int kTcTmemCols = 128;
constexpr int kTcSmem = 1024 + kTcStages * kTcStageBytes + 256;
constexpr int64_t kTcSms = 148;                    // SM count the split plan is tuned for (B200)

struct TcPlan {
  int64_t ntiles, kblocks, kbps, nsplit;
  size_t bw_bytes;  // workspace bytes of Bw, rounded to 1 KB
};

static TcPlan tc_plan(int64_t T, int64_t H) {
  TcPlan p;
  const int64_t K = 4 * H;
  p.ntiles = (T + kTcM - 1) / kTcM;
  p.kblocks = (K + kTcKB - 1) / kTcKB;
  // Splits per tile: at least 3 waves of CTAs (one CTA per SM); then the fewest splits whose last
  // wave is at least 90% full (each CTA's pipeline fill is exposed, so longer CTAs are better),
  // else the fullest last wave seen.
  const int64_t ns_min = (3 * kTcSms + p.ntiles - 1) / p.ntiles;
  int64_t best_ns = ns_min > p.kblocks ? p.kblocks : (ns_min < 1 ? 1 : ns_min);
  double best_eff = -1.0;
  for (int64_t ns = best_ns; ns <= ns_min + 16 && ns <= p.kblocks; ++ns) {
    const int64_t kbps = (p.kblocks + ns - 1) / ns;
    const int64_t nsplit = (p.kblocks + kbps - 1) / kbps;
    const int64_t ctas = nsplit * p.ntiles;
    const int64_t waves = (ctas + kTcSms - 1) / kTcSms;
    const double eff = static_cast<double>(ctas) / static_cast<double>(waves * kTcSms);
    if (eff > best_eff + 1e-9) {
      best_eff = eff;
      best_ns = ns;
    }
    if (eff >= 0.9) break;
  }
  p.kbps = (p.kblocks + best_ns - 1) / best_ns;
  p.nsplit = (p.kblocks + p.kbps - 1) / p.kbps;
  p.bw_bytes = (static_cast<size_t>(kTcN) * K * 2 + 1023) / 1024 * 1024;
  return p;
}

bool pre_tc_supported(int64_t T, int64_t H) {
  // TMA needs 16-byte global strides: rows of R (8H bytes) and of Bw (8H bytes).
  return T >= 1 && H >= 2 && H % 2 == 0 && tc_plan(T, H).nsplit <= 65535 &&
         (T + kTcM - 1) / kTcM <= 0x7fffffff;
}

size_t pre_tc_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0 || H % 2 != 0) return 0;
  const TcPlan p = tc_plan(T, H);
  return p.bw_bytes + static_cast<size_t>(p.nsplit) * static_cast<size_t>(T) * 32 * sizeof(float);
}

// ------------------------------------------------------------------------------ device helpers

__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M = 128, N = 80.
constexpr uint32_t kTcIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kTcN >> 3) << 17) |
                              (static_cast<uint32_t>(kTcM >> 4) << 24);

__device__ __forceinline__ void umma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kTcIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ------------------------------------------------------------------------------ kernels

// hc_fn [K][24] fp32 -> Bw [80][K] bf16: rows j, 24+j, 48+j hold the hi, mid, lo terms of column
// j (w = hi + mid + lo exactly: each remainder is exact in fp32 and the last fits 8 bits); rows
// 72..79 are zero.
__global__ void __launch_bounds__(256) pre_tc_split_kernel(const float* __restrict__ W,
                                                           uint16_t* __restrict__ Bw, int64_t K) {
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < K;
       k += (int64_t)gridDim.x * blockDim.x) {
#pragma unroll 4
    for (int j = 0; j < kMix; ++j) {
      const float w = W[k * kMix + j];
      const uint16_t hi = f32_to_bf16(w);
      const float r1 = w - bf16_to_f32(hi);
      const uint16_t mid = f32_to_bf16(r1);
      const float r2 = r1 - bf16_to_f32(mid);
      const uint16_t lo = f32_to_bf16(r2);
      Bw[j * K + k] = hi;
      Bw[(kMix + j) * K + k] = mid;
      Bw[(2 * kMix + j) * K + k] = lo;
    }
#pragma unroll
    for (int j = 3 * kMix; j < kTcN; ++j) Bw[j * K + k] = 0;
  }
}

__global__ void __launch_bounds__(kTcThreads, 1) pre_tc_proj_kernel(
    const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmB,
    float* __restrict__ part, int64_t T, int kblocks, int kbps) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kTcStages * kTcStageBytes);
  uint64_t* empty = full + kTcStages;
  uint64_t* accum = empty + kTcStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(accum + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = blockIdx.x;
  const int split = blockIdx.y;
  const int kb0 = split * kbps;
  const int nkb = min(kblocks, kb0 + kbps) - kb0;  // >= 1 by the plan

  if (threadIdx.x == 0) {
    for (int s = 0; s < kTcStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA commit + one arrival per sum-of-squares warp
    }
    mbar_init(accum, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kTcTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    if (lane == 0) {
      int issued = 0;
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kTcStages;
        const uint32_t ph = static_cast<uint32_t>(i / kTcStages) & 1u;
        if (i >= kTcStages && !mbar_wait(&empty[s], ph ^ 1u, 10)) {
          ok = false;
          break;
        }
        uint8_t* st = smem + s * kTcStageBytes;
        mbar_arrive_expect_tx(&full[s], kTcStageBytes);
        tma_load_2d(st, &tmR, (kb0 + i) * kTcKB, tile * kTcM, &full[s]);
        tma_load_2d(st + kTcABytes, &tmB, (kb0 + i) * kTcKB, 0, &full[s]);
        ++issued;
      }
      if (!ok) {  // do not leave while copies into shared memory are in flight
        for (int i = issued - kTcStages; i < issued; ++i)
          if (i >= 0)
            mbar_wait(&full[i % kTcStages], static_cast<uint32_t>(i / kTcStages) & 1u, 15);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      bool ok = true;
      for (int i = 0; i < nkb; ++i) {
        const int s = i % kTcStages;
        const uint32_t ph = static_cast<uint32_t>(i / kTcStages) & 1u;
        if (!mbar_wait(&full[s], ph, 11)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a = smem_u32(smem + s * kTcStageBytes);
        const uint64_t adesc = sw128_desc(a);
        const uint64_t bdesc = sw128_desc(a + kTcABytes);
#pragma unroll
        for (int k = 0; k < kTcKB / 16; ++k)  // +32 bytes along the swizzled row per K=16 step
          umma_bf16(tmem, adesc + 2 * k, bdesc + 2 * k, (i > 0 || k > 0) ? 1u : 0u);
        umma_commit(&empty[s]);
      }
      umma_commit(accum);
      if (!ok) mbar_wait(accum, 0, 14);
    }
  } else {
    // Warps 2..5: TMEM lane quarter q = warp % 4 holds accumulator rows 32q..32q+31; the same
    // thread sums the squares of that row.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    float ss0 = 0.f, ss1 = 0.f;
    bool ok = true;
    for (int i = 0; i < nkb; ++i) {
      const int s = i % kTcStages;
      const uint32_t ph = static_cast<uint32_t>(i / kTcStages) & 1u;
      // Every lane waits; the warp continues only if all of them saw the stage (warp-uniform, so
      // the __syncwarp and the .sync.aligned TMEM loads below are never reached divergently).
      if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, 12))) {
        ok = false;
        break;
      }
      // Row `row` of the swizzled tile is its own 128 contiguous bytes (chunks permuted within
      // it), and a sum does not depend on element order. Each lane starts at a different 16-byte
      // chunk, so the 8 lanes of a load phase hit 8 different bank groups.
      const uint4* rp = reinterpret_cast<const uint4*>(smem + s * kTcStageBytes + row * 128);
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint4 v = rp[c ^ (lane & 7)];
        const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float a = bf16_lo(u[e]), b = bf16_hi(u[e]);
          ss0 = fmaf(a, a, ss0);
          ss1 = fmaf(b, b, ss1);
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
    if (ok && __all_sync(0xffffffffu, mbar_wait(accum, 0, 13))) {
      tc_fence_after();
      uint32_t d[5][16];
      const uint32_t tbase = tmem + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
      for (int c = 0; c < 5; ++c) tmem_ld16(tbase + c * 16, d[c]);
      tmem_wait_ld();
      const int64_t t = static_cast<int64_t>(tile) * kTcM + row;
      if (t < T) {
        float raw[kMix];
#pragma unroll
        for (int j = 0; j < kMix; ++j) {
          const float hi = __uint_as_float(d[j / 16][j % 16]);
          const float mid = __uint_as_float(d[(kMix + j) / 16][(kMix + j) % 16]);
          const float lo = __uint_as_float(d[(2 * kMix + j) / 16][(2 * kMix + j) % 16]);
          raw[j] = (lo + mid) + hi;
        }
        float4* rec = reinterpret_cast<float4*>(part + (static_cast<int64_t>(split) * T + t) * 32);
#pragma unroll
        for (int v = 0; v < 6; ++v)
          rec[v] = make_float4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
        rec[6] = make_float4(ss0 + ss1, 0.f, 0.f, 0.f);
      }
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kTcTmemCols)
                 : "memory");
  }
}

// Coefficients from the split records [split][t][32] (raw[0..23], ss): one token per lane quad,
// 8 tokens per warp. Lane r of a quad sums, over the splits in order, the components it needs
// (pre r, post r, comb row r, ss) and runs its row of the Sinkhorn.
__global__ void __launch_bounds__(256) pre_tc_coef_kernel(const float* __restrict__ part,
                                                          int64_t nsplit,
                                                          const float* __restrict__ scale,
                                                          const float* __restrict__ base,
                                                          float* __restrict__ pre,
                                                          float* __restrict__ post,
                                                          float* __restrict__ comb, int64_t T,
                                                          int64_t K, FinishParams fp) {
  const int lane = threadIdx.x & 31;
  const int r = lane & 3;
  const int64_t t = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 2;
  const bool live = t < T;
  const int64_t tt = live ? t : 0;
  float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, gc = g0, g6 = g0;
  for (int64_t s = 0; s < nsplit; ++s) {
    const float4* rec = reinterpret_cast<const float4*>(part + (s * T + tt) * 32);
    const float4 a0 = __ldg(rec), a1 = __ldg(rec + 1), ac = __ldg(rec + 2 + r), a6 = __ldg(rec + 6);
    g0.x += a0.x, g0.y += a0.y, g0.z += a0.z, g0.w += a0.w;
    g1.x += a1.x, g1.y += a1.y, g1.z += a1.z, g1.w += a1.w;
    gc.x += ac.x, gc.y += ac.y, gc.z += ac.z, gc.w += ac.w;
    g6.x += a6.x;
  }
  const float p0[4] = {g0.x, g0.y, g0.z, g0.w};
  const float p1[4] = {g1.x, g1.y, g1.z, g1.w};
  const float rstd =
      __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(g6.x, static_cast<float>(K)) + fp.rms_eps));
  const float lp = fmaf(p0[r] * rstd, __ldg(scale), __ldg(base + r));
  const float lq = fmaf(p1[r] * rstd, __ldg(scale + 1), __ldg(base + 4 + r));
  const float s2 = __ldg(scale + 2);
  float cr[4] = {fmaf(gc.x * rstd, s2, __ldg(base + 8 + 4 * r)),
                 fmaf(gc.y * rstd, s2, __ldg(base + 9 + 4 * r)),
                 fmaf(gc.z * rstd, s2, __ldg(base + 10 + 4 * r)),
                 fmaf(gc.w * rstd, s2, __ldg(base + 11 + 4 * r))};
  sinkhorn_quad(cr, fp.iters, fp.sinkhorn_eps);  // every lane takes part
  if (live) {
    pre[t * 4 + r] = sigmoidf_ieee(lp) + fp.pre_eps;
    post[t * 4 + r] = fp.post_mult * sigmoidf_ieee(lq);
    float* dst = comb + t * 16 + r * 4;
    dst[0] = cr[0], dst[1] = cr[1], dst[2] = cr[2], dst[3] = cr[3];
  }
}

// y = bf16_rn(sum_i pre_i * R_i): one thread per (token, 8 columns), a streaming pass (R read once,
// y written once). Requires H % 8 == 0 and 16-byte aligned R and y.
__global__ void __launch_bounds__(256) pre_agg_vec8_kernel(const uint16_t* __restrict__ R,
                                                           const float* __restrict__ pre,
                                                           uint16_t* __restrict__ y, int64_t T,
                                                           int64_t H8) {
  const int64_t total = T * H8;
  const int64_t H = H8 * 8;
  for (int64_t u = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; u < total;
       u += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = u / H8;
    const int64_t v = u - t * H8;
    const uint16_t* rr = R + t * 4 * H + v * 8;
    uint4 rv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) rv[i] = ld_stream_ro(rr + i * H);
    const float4 p4 = __ldg(reinterpret_cast<const float4*>(pre + t * 4));
    const uint32_t* r0 = &rv[0].x;
    const uint32_t* r1 = &rv[1].x;
    const uint32_t* r2 = &rv[2].x;
    const uint32_t* r3 = &rv[3].x;
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float lo = p4.x * bf16_lo(r0[e]);
      lo = fmaf(p4.y, bf16_lo(r1[e]), lo);
      lo = fmaf(p4.z, bf16_lo(r2[e]), lo);
      lo = fmaf(p4.w, bf16_lo(r3[e]), lo);
      float hi = p4.x * bf16_hi(r0[e]);
      hi = fmaf(p4.y, bf16_hi(r1[e]), hi);
      hi = fmaf(p4.z, bf16_hi(r2[e]), hi);
      hi = fmaf(p4.w, bf16_hi(r3[e]), hi);
      o[e] = pack_bf16x2(lo, hi);
    }
    st_plain(y + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// ------------------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_tiled() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// 2-D bf16 tensor map over a row-major [rows][cols] matrix, box [box_rows][64], 128-byte swizzle,
// out-of-range elements read as zero.
static bool make_map(CUtensorMap* m, const void* base, int64_t cols, int64_t rows, int box_rows) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(cols) * 2};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(kTcKB), static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int launch_pre_tc(const PreArgs& a, cudaStream_t s) {
  const TcPlan plan = tc_plan(a.T, a.H);
  const int64_t K = 4 * a.H;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  uint16_t* Bw = reinterpret_cast<uint16_t*>(ws);
  float* part = reinterpret_cast<float*>(ws + plan.bw_bytes);

  CUtensorMap mR, mB;
  if (!make_map(&mR, a.R, K, a.T, kTcM) || !make_map(&mB, Bw, K, kTcN, kTcN)) return -4;

  static bool attr_set[64] = {};
  const int dev = current_device();
  if (dev < 0) return -4;
  if (!attr_set[dev]) {
    if (cudaFuncSetAttribute(pre_tc_proj_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             kTcSmem) != cudaSuccess)
      return -4;
    attr_set[dev] = true;
  }

  const int64_t sb = (K + 255) / 256;
  const int split_blocks = static_cast<int>(sb < 4096 ? sb : 4096);
  pre_tc_split_kernel<<<split_blocks, 256, 0, s>>>(a.hc_fn, Bw, K);
  note_launches(1);
  if (cudaGetLastError() != cudaSuccess) return -4;

  const dim3 grid(static_cast<unsigned>(plan.ntiles), static_cast<unsigned>(plan.nsplit));
  pre_tc_proj_kernel<<<grid, kTcThreads, kTcSmem, s>>>(mR, mB, part, a.T,
                                                       static_cast<int>(plan.kblocks),
                                                       static_cast<int>(plan.kbps));
  note_launches(1);
  if (cudaGetLastError() != cudaSuccess) return -4;

  const FinishParams fp{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};
  const bool vec = aligned16(a.R) && aligned16(a.y) && aligned16(a.pre) && (a.H % 8 == 0);
  if (vec) {
    // Coefficients for all tokens, then one streaming pass for y.
    const int64_t cb = (4 * a.T + 255) / 256;
    if (cb > 0x7fffffff) return -5;
    pre_tc_coef_kernel<<<static_cast<unsigned>(cb), 256, 0, s>>>(
        part, plan.nsplit, a.hc_scale, a.hc_base, a.pre, a.post, a.comb, a.T, 4 * a.H, fp);
    note_launches(1);
    if (cudaGetLastError() != cudaSuccess) return -4;
    const int64_t units = a.T * (a.H / 8);
    int64_t ab = (units + 255) / 256;
    const int64_t cap = static_cast<int64_t>(device_sm_count()) * 16;
    if (ab > cap) ab = cap;
    pre_agg_vec8_kernel<<<static_cast<unsigned>(ab), 256, 0, s>>>(a.R, a.pre, a.y, a.T, a.H / 8);
  } else {
    const int64_t nhb = (a.H + kAggCols - 1) / kAggCols;
    if (a.T > 0x7fffffff || 1 + nhb > 65535) return -5;
    const dim3 g2(static_cast<unsigned>(a.T), static_cast<unsigned>(1 + nhb));
    pre_cc_finish_kernel<false><<<g2, 256, 0, s>>>(a.R, part, plan.nsplit, a.hc_scale,
                                                   a.hc_base, a.y, a.pre, a.post, a.comb, a.T,
                                                   a.H, fp);
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace mhc
