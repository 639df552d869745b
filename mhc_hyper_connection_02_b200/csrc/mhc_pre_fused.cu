// mHC pre-map as one persistent kernel: projection on tcgen05, sum of squares, cross-CTA
// reduction, coefficients (gates, Sinkhorn) and aggregate. Streaming R from HBM never waits for
// the reduction.
//
// Work split. The hidden dimension is cut into 64-column slices; CTA c of a group owns q
// consecutive slices (all four streams of them: 4q blocks of the flattened K = 4H, so it can also
// form y on those columns) and keeps that part of the split hc_fn operand (Bw, bf16 x3, see
// mhc_pre_tc.cu) resident in shared memory. A group of NSG CTAs covers all of H; G groups take
// token tiles of 128 round robin. Per tile, inside each CTA:
//
//   warp 0      TMA, projection ring: R block [128 tokens x 64 columns] of one stream per 16 KB
//               stage (128-byte swizzle, the MMA operand layout).
//   warp 1      tcgen05.mma M=128 N=80 K=16 into one of two TMEM accumulators.
//   warps 2-5   sum of squares of each token row from the projection stage; after the tile the
//               accumulator (tcgen05.ld) becomes the split record [group][tile ring][token][c][32]
//               = raw[24], ss; release-increment count[tile].
//   warps 6-8   one tile in three each: once count[tile] == NSG, sum the NSG records of this
//               CTA's tokens (t = c, c + NSG, ...) in a fixed order, write the pre gates and
//               release-increment ready[tile]; then post and comb (Sinkhorn), off the critical path.
//   warp 9      releases count[tile] once the record warps have written (one gpu-scope fence per
//               tile, so the record warps never stall on it).
//   warps 10-15 once ready[tile] == NSG: y = sum_i pre_i * R_i on this CTA's columns, re-reading
//               the tile with ordinary 16-byte loads. It was streamed a few microseconds earlier, so
//               these hit L2, and they use the SM's load path rather than the TMA engine, whose
//               per-SM rate the projection stream already uses up.
//
// Counters are zeroed by a kernel launched just before. All CTAs are co-resident (cooperative
// launch, one CTA per SM) and every wait is bounded by time: on expiry the kernel records
// MHC_ERR_TIMEOUT in the status word and winds down instead of waiting forever.
//
// "FlashInfer mHC module deep dive" §3.4 (per-token phases: sum of squares and rstd, gates,
// softmax and Sinkhorn rounds, vec8 aggregate) and §3.3 (split reduction of dot_mix / sqrsum);
// glm5next_mhc.rs glm_hc_pre (mix then finish).
#include <cuda.h>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kFuM = 128;
constexpr int kFuN = 80;
constexpr int kFuHS = 64;                        // columns per slice
constexpr int kFuPBytes = kFuM * kFuHS * 2;      // 16384: projection stage
constexpr int kFuBBytes = kFuN * kFuHS * 2;      // 10240: one Bw block
constexpr int kFuMaxQ = 2;
constexpr int kFuRing = 8;                       // tiles of split records in flight
constexpr int kFuRec = 32;                       // floats per record
constexpr int kFuCoefWarps = 3;                  // warps 6..8
constexpr int kFuRelWarp = 9;
constexpr int kFuAggWarp0 = 10;                  // warps 10..15
constexpr int kFuAggThreads = 6 * 32;
constexpr int kFuThreads = 512;
constexpr int kFuTmemCols = 256;                 // two accumulators at columns 0 and 128
constexpr int kFuSmsPlan = 148;                  // SM count the workspace plan assumes (B200)
// Slices per CTA are chosen so that a group has at most this many CTAs: two tile groups then run
// side by side on 148 SMs, a token's records are fewer, and each CTA has twice the time per tile.
constexpr int kFuGroupCtas = 74;
constexpr int kFuTot = 28;                       // floats per token total in shared memory
constexpr int kFuBarBytes = 512;                // mbarriers and the TMEM address word
constexpr int kFuMisc = kFuBarBytes + kFuCoefWarps * 8 * kFuTot * 4;  // + coefficient scratch

// Ring depths by slices per CTA (shared memory: 1 KB alignment slack + rings + Bw + misc).
__host__ __device__ constexpr int fu_pstages(int q) { return q == 1 ? 11 : 8; }

struct FuPlan {
  int64_t ns;     // 64-column slices
  int64_t q;      // slices per CTA
  int64_t nsg;    // CTAs per group
  int64_t ntiles;
  int64_t gmax;   // most tile groups a launch may use (each has its own record ring)
  size_t bw_bytes, cnt_off, part_off, total;
};

static FuPlan fu_plan(int64_t T, int64_t H) {
  FuPlan p;
  p.ns = (H + kFuHS - 1) / kFuHS;
  p.q = (p.ns + kFuGroupCtas - 1) / kFuGroupCtas;
  if (p.q > kFuMaxQ) p.q = (p.ns + kFuSmsPlan - 1) / kFuSmsPlan;  // wide H: one group
  p.nsg = (p.ns + p.q - 1) / p.q;
  p.ntiles = (T + kFuM - 1) / kFuM;
  p.gmax = kFuSmsPlan / p.nsg;
  if (p.gmax > p.ntiles) p.gmax = p.ntiles;
  if (p.gmax < 1) p.gmax = 1;
  p.bw_bytes = (static_cast<size_t>(kFuN) * 4 * H * 2 + 1023) / 1024 * 1024;
  p.cnt_off = p.bw_bytes;
  p.part_off = p.cnt_off + (static_cast<size_t>(2 * p.ntiles) * 4 + 255) / 256 * 256;
  p.total = p.part_off + static_cast<size_t>(p.gmax) * kFuRing * kFuM * p.nsg * kFuRec * 4;
  return p;
}

static int fu_smem_bytes(int q) {
  return 1024 + fu_pstages(q) * kFuPBytes + 4 * q * kFuBBytes + kFuMisc;
}

bool pre_fused_supported(int64_t T, int64_t H) {
  if (T < 1 || H < 8 || H % 8 != 0) return false;
  const FuPlan p = fu_plan(T, H);
  // At least 8 CTAs per group keeps a CTA's tokens per tile within two batches of 8.
  return p.q <= kFuMaxQ && p.nsg >= 8 && p.ntiles <= (int64_t(1) << 30);
}

size_t pre_fused_workspace_bytes(int64_t T, int64_t H) {
  if (!pre_fused_supported(T, H)) return 0;
  return fu_plan(T, H).total;
}

// ------------------------------------------------------------------------------ device helpers

__device__ __forceinline__ void tma_load_3d(void* dst, const CUtensorMap* map, int x, int y, int z,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}
// Named barrier that also ORs a predicate over the participating threads (every thread gets the
// same answer, so decisions taken on it are uniform and barrier sequences stay matched).
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
// Release increment: everything this thread has observed (including, through CTA-scope
// synchronisation, other threads' stores) is visible at gpu scope before the add.
__device__ __forceinline__ void red_release_add(int* p, int v) {
  asm volatile("fence.acq_rel.gpu;\n\tred.relaxed.gpu.global.add.s32 [%0], %1;" ::"l"(p), "r"(v)
               : "memory");
}
__device__ __forceinline__ bool status_set() {
  return *reinterpret_cast<volatile int*>(&g_device_status) != 0;
}

// Waits until *p >= target; false on timeout (or once another wait has timed out).
__device__ __noinline__ bool wait_count(const int* p, int target, int where) {
  if (ld_acquire(p) >= target) return true;
  if (status_set()) return false;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(20);
    if (ld_acquire(p) >= target) return true;
    if ((i & 63u) == 0) {
      if (status_set()) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        report_timeout(where);
        return false;
      }
    }
  }
}

struct FuArgs {
  const uint16_t* R;
  const float* scale;
  const float* base;
  uint16_t* y;
  float* pre;
  float* post;
  float* comb;
  int* cnt;      // [ntiles]
  int* ready;    // [ntiles]
  float* part;   // [groups][kFuRing][128][nsg][32]
  int64_t T, H;
  int ntiles, nsg, q, groups;
  FinishParams fp;
};

// Sums the NSG records of one token into tot (28 floats in shared memory). The token's records
// are contiguous (NSG x 128 bytes); lane l adds float4 number l, l+32, ...: component group l % 8
// of records l/8, l/8 + 4, ... in increasing order, then a fixed xor tree joins the four lanes of
// each group. The order is fixed, so every run gives the same sums.
__device__ __forceinline__ void fu_reduce_token(const float* recs_f, int nsg, float* tot) {
  const int lane = threadIdx.x & 31;
  const float4* recs = reinterpret_cast<const float4*>(recs_f);
  const int nf4 = nsg * (kFuRec / 4);
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  constexpr int kU = 14;  // loads in flight per lane
  for (int m0 = lane; m0 < nf4; m0 += 32 * kU) {
    float4 v[kU];
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      const int m = m0 + 32 * u;
      v[u] = m < nf4 ? __ldcg(recs + m) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < kU; ++u) {
      acc.x += v[u].x;
      acc.y += v[u].y;
      acc.z += v[u].z;
      acc.w += v[u].w;
    }
  }
#pragma unroll
  for (int sh = 8; sh <= 16; sh <<= 1) {
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, sh);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, sh);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, sh);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, sh);
  }
  if (lane < kFuTot / 4) reinterpret_cast<float4*>(tot)[lane] = acc;
}

__global__ void __launch_bounds__(kFuThreads, 1) pre_fused_kernel(
    const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmB,
    const FuArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  const int nP = fu_pstages(a.q);
  const int nkb = 4 * a.q;  // projection blocks (and aggregate stages) per tile
  uint8_t* pring = smem;
  uint8_t* bres = pring + nP * kFuPBytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(bres + nkb * kFuBBytes);
  uint64_t* pfull = bars;             // [11]
  uint64_t* pempty = bars + 11;       // [11]
  uint64_t* bfull = bars + 22;
  uint64_t* dfull = bars + 23;        // [2]
  uint64_t* dempty = bars + 25;       // [2]
  uint64_t* mma_done = bars + 27;
  uint64_t* recdone = bars + 28;      // [2] record warps -> warp 15
  uint64_t* recfree = bars + 30;      // [2] warp 15 -> record warps
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 32);
  float* coef_smem = reinterpret_cast<float*>(reinterpret_cast<uint8_t*>(bars) + kFuBarBytes);
  static_assert(33 * 8 <= kFuBarBytes, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int c = blockIdx.x % a.nsg;  // slice group within the tile group
  const int g = blockIdx.x / a.nsg;  // tile group
  const int h0 = c * a.q * kFuHS;    // first column of this CTA
  const int64_t K = 4 * a.H;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nP; ++s) {
      mbar_init(&pfull[s], 1);
      mbar_init(&pempty[s], 1 + 4);  // MMA commit + one arrival per sum-of-squares warp
    }
    mbar_init(bfull, 1);
    for (int d = 0; d < 2; ++d) {
      mbar_init(&dfull[d], 1);
      mbar_init(&dempty[d], 4);
    }
    mbar_init(mma_done, 1);
    for (int d = 0; d < 2; ++d) {
      mbar_init(&recdone[d], 4);
      mbar_init(&recfree[d], 1);
    }
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kFuTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  if (warp == 0) {
    // ---------------------------------------------------------------- projection TMA
    if (lane == 0) {
      mbar_arrive_expect_tx(bfull, nkb * kFuBBytes);
      for (int kb = 0; kb < nkb; ++kb)
        tma_load_3d(bres + kb * kFuBBytes, &tmB, h0 + (kb >> 2) * kFuHS, kb & 3, 0, bfull);
      int64_t n = 0;
      bool ok = true;
      for (int j = g; j < a.ntiles && ok; j += a.groups) {
        for (int kb = 0; kb < nkb; ++kb, ++n) {
          const int s = static_cast<int>(n % nP);
          const uint32_t ph = static_cast<uint32_t>(n / nP) & 1u;
          if (n >= nP && !mbar_wait(&pempty[s], ph ^ 1u, 20)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&pfull[s], kFuPBytes);
          tma_load_3d(pring + s * kFuPBytes, &tmR, h0 + (kb >> 2) * kFuHS, kb & 3, j * kFuM,
                      &pfull[s]);
        }
      }
      // Never leave with copies into shared memory in flight.
      mbar_wait(bfull, 0, 21);
      for (int64_t i = n - nP; i < n; ++i)
        if (i >= 0) mbar_wait(&pfull[i % nP], static_cast<uint32_t>(i / nP) & 1u, 22);
    }
  } else if (warp == 1) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      bool ok = mbar_wait(bfull, 0, 23);
      int64_t n = 0;
      int it = 0;
      for (int j = g; j < a.ntiles && ok; j += a.groups, ++it) {
        const int d = it & 1;
        if (it >= 2 && !mbar_wait(&dempty[d], static_cast<uint32_t>((it >> 1) - 1) & 1u, 24)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dtm = tmem + static_cast<uint32_t>(d * 128);
        for (int kb = 0; kb < nkb; ++kb, ++n) {
          const int s = static_cast<int>(n % nP);
          const uint32_t ph = static_cast<uint32_t>(n / nP) & 1u;
          if (!mbar_wait(&pfull[s], ph, 25)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t adesc = sw128_desc(smem_u32(pring + s * kFuPBytes));
          const uint64_t bdesc = sw128_desc(smem_u32(bres + kb * kFuBBytes));
#pragma unroll
          for (int k = 0; k < kFuHS / 16; ++k)
            umma_bf16(dtm, adesc + 2 * k, bdesc + 2 * k, (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit(&pempty[s]);
        }
        umma_commit(&dfull[d]);
      }
      // Every issued MMA has finished before TMEM is released.
      umma_commit(mma_done);
      mbar_wait(mma_done, 0, 31);
    }
  } else if (warp < 6) {
    // ---------------------------------------------------------------- sum of squares + records
    // Loops never leave early: after a failed wait a thread only skips work, so the four warps
    // always meet the same named barriers; the barrier's OR makes a failure uniform.
    const int qd = warp & 3;
    const int row = qd * 32 + lane;
    int64_t n = 0;
    int it = 0;
    bool dead = false;
    for (int j = g; j < a.ntiles; j += a.groups, ++it) {
      float ss0 = 0.f, ss1 = 0.f;
      for (int kb = 0; kb < nkb; ++kb, ++n) {
        const int s = static_cast<int>(n % nP);
        const uint32_t ph = static_cast<uint32_t>(n / nP) & 1u;
        if (!dead) dead = !__all_sync(0xffffffffu, mbar_wait(&pfull[s], ph, 26));
        if (dead) continue;
        // Row `row` of the swizzled block is its own 128 contiguous bytes (chunks permuted within
        // it), and a sum does not depend on element order. Each lane starts at a different 16-byte
        // chunk, so the 8 lanes of a load phase hit 8 different bank groups.
        const uint4* rp = reinterpret_cast<const uint4*>(pring + s * kFuPBytes + row * 128);
#pragma unroll
        for (int cc = 0; cc < 8; ++cc) {
          const uint4 v = rp[cc ^ (lane & 7)];
          const uint32_t u[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float x0 = bf16_lo(u[e]), x1 = bf16_hi(u[e]);
            ss0 = fmaf(x0, x0, ss0);
            ss1 = fmaf(x1, x1, ss1);
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&pempty[s]);
      }
      const int d = it & 1;
      if (!dead)
        dead = !__all_sync(0xffffffffu,
                           mbar_wait(&dfull[d], static_cast<uint32_t>(it >> 1) & 1u, 27));
      uint32_t dr[5][16];
      if (!dead) {
        tc_fence_after();
        const uint32_t tb =
            tmem + static_cast<uint32_t>(d * 128) + (static_cast<uint32_t>(qd * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < 5; ++cc) tmem_ld16(tb + cc * 16, dr[cc]);
        tmem_wait_ld();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&dempty[d]);
      }
      // Ring slot reuse: the records of tile j - kFuRing*groups must have been consumed.
      bool w = true;
      if (it >= kFuRing && threadIdx.x == 64 && !dead)
        w = wait_count(&a.ready[j - kFuRing * a.groups], a.nsg, 28);
      dead = named_bar_or(1, 128, dead || !w);
      const int64_t t = static_cast<int64_t>(j) * kFuM + row;
      if (!dead && t < a.T) {
        const int64_t slot = static_cast<int64_t>(g) * kFuRing + it % kFuRing;
        float* rec = a.part + ((slot * kFuM + row) * a.nsg + c) * kFuRec;
        float raw[kMix];
#pragma unroll
        for (int jj = 0; jj < kMix; ++jj) {
          const float hi = __uint_as_float(dr[jj / 16][jj % 16]);
          const float mi = __uint_as_float(dr[(kMix + jj) / 16][(kMix + jj) % 16]);
          const float lo = __uint_as_float(dr[(2 * kMix + jj) / 16][(2 * kMix + jj) % 16]);
          raw[jj] = (lo + mi) + hi;
        }
        float4* r4 = reinterpret_cast<float4*>(rec);
#pragma unroll
        for (int v = 0; v < 6; ++v)
          r4[v] = make_float4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
        r4[6] = make_float4(ss0 + ss1, 0.f, 0.f, 0.f);
      }
      // Hand the tile to warp 15, which releases count[tile]. Its 2-slot ring is guarded by
      // recfree so that a slot's phase is consumed before it is armed again.
      const int rs = it & 1;
      if (it >= 2 && !dead)
        dead = !__all_sync(0xffffffffu,
                           mbar_wait(&recfree[rs], static_cast<uint32_t>((it >> 1) - 1) & 1u, 36));
      __syncwarp();
      if (lane == 0) mbar_arrive(&recdone[rs]);
    }
  } else if (warp < 6 + kFuCoefWarps) {
    // ---------------------------------------------------------------- coefficients
    // Warp cw takes every kFuCoefWarps-th tile of this CTA; no barrier ties the coefficient warps
    // together. For a tile: sum the records of this CTA's tokens (at most 16: NSG >= 8), write the
    // pre gates, signal ready (the aggregate needs only those), then post and comb. Lane quad k
    // handles token k of a batch of 8; lane r of the quad owns row r of comb.
    const int cw = warp - 6;
    float* tot_s = coef_smem + cw * 8 * kFuTot;
    int it = 0;
    bool dead = false;
    for (int j = g; j < a.ntiles; j += a.groups, ++it) {
      if (it % kFuCoefWarps != cw) continue;
      bool w = true;
      if (lane == 0 && !dead) w = wait_count(&a.cnt[j], a.nsg, 29);
      dead = dead || !__all_sync(0xffffffffu, w);
      const int64_t slot = static_cast<int64_t>(g) * kFuRing + it % kFuRing;
      int ntok = 0;  // this CTA's tokens in the tile: tl = c + k*NSG
      for (int tl = c; tl < kFuM && static_cast<int64_t>(j) * kFuM + tl < a.T; tl += a.nsg) ++ntok;
      const int nbatch = (ntok + 7) / 8;
      for (int pass = 0; pass < 2 && !dead; ++pass) {
        for (int b = 0; b < nbatch; ++b) {
          const int nk = min(8, ntok - 8 * b);
          // A single batch keeps its sums from the first pass.
          if (pass == 0 || nbatch > 1) {
            for (int k = 0; k < nk; ++k) {
              const int tl = c + (8 * b + k) * a.nsg;
              fu_reduce_token(a.part + (slot * kFuM + tl) * a.nsg * kFuRec, a.nsg,
                              tot_s + k * kFuTot);
            }
            __syncwarp();
          }
          const int k = lane >> 2;
          const int r = lane & 3;
          const bool live = k < nk;
          const float* tt = tot_s + (live ? k : 0) * kFuTot;
          const int64_t t = static_cast<int64_t>(j) * kFuM + c + (8 * b + (live ? k : 0)) * a.nsg;
          const float rstd = __fdiv_rn(
              1.0f, __fsqrt_rn(__fdiv_rn(tt[24], static_cast<float>(K)) + a.fp.rms_eps));
          if (pass == 0) {
            const float lp = fmaf(tt[r] * rstd, __ldg(a.scale), __ldg(a.base + r));
            if (live) a.pre[t * 4 + r] = sigmoidf_ieee(lp) + a.fp.pre_eps;
          } else {
            const float lq = fmaf(tt[4 + r] * rstd, __ldg(a.scale + 1), __ldg(a.base + 4 + r));
            float cr[4];
#pragma unroll
            for (int nn = 0; nn < 4; ++nn)
              cr[nn] = fmaf(tt[8 + 4 * r + nn] * rstd, __ldg(a.scale + 2),
                            __ldg(a.base + 8 + 4 * r + nn));
            sinkhorn_quad(cr, a.fp.iters, a.fp.sinkhorn_eps);  // every lane takes part
            if (live) {
              a.post[t * 4 + r] = a.fp.post_mult * sigmoidf_ieee(lq);
              *reinterpret_cast<float4*>(a.comb + t * 16 + r * 4) =
                  make_float4(cr[0], cr[1], cr[2], cr[3]);
            }
          }
          __syncwarp();
        }
        if (pass == 0) {
          __syncwarp();
          if (lane == 0) red_release_add(&a.ready[j], 1);
        }
      }
    }
  } else if (warp >= kFuAggWarp0) {
    // ---------------------------------------------------------------- aggregate
    // Units of 8 columns: e = 8q * token + column group. Thread `at` takes units at, at + 192, ...
    // in batches of 4 (all loads of a batch in flight before any use), so a warp reads 4 tokens x
    // 128 q bytes of each stream per load instruction.
    const int at = threadIdx.x - kFuAggWarp0 * 32;
    const int upt = 8 * a.q;
    const int units = kFuM * upt;
    bool dead = false;
    for (int j = g; j < a.ntiles; j += a.groups) {
      bool w = true;
      if (at == 0 && !dead) w = wait_count(&a.ready[j], a.nsg, 30);
      dead = named_bar_or(3, kFuAggThreads, dead || !w);
      if (dead) continue;
      constexpr int kB = 4;
      for (int e0 = at; e0 < units; e0 += kB * kFuAggThreads) {
        uint4 r[kB][4];
        float4 p4[kB];
        int64_t tok[kB];
        int hc[kB];
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          const int e = e0 + u * kFuAggThreads;
          const int tl = e / upt;
          const int hcol = h0 + (e - tl * upt) * 8;
          const int64_t t = static_cast<int64_t>(j) * kFuM + tl;
          hc[u] = hcol;
          tok[u] = (e < units && t < a.T && hcol < a.H) ? t : -1;
          if (tok[u] < 0) continue;
          p4[u] = __ldcg(reinterpret_cast<const float4*>(a.pre + t * 4));
          const uint16_t* rr = a.R + t * 4 * a.H + hcol;
#pragma unroll
          for (int i = 0; i < 4; ++i) r[u][i] = __ldg(reinterpret_cast<const uint4*>(rr + i * a.H));
        }
#pragma unroll
        for (int u = 0; u < kB; ++u) {
          if (tok[u] < 0) continue;
          const float p[4] = {p4[u].x, p4[u].y, p4[u].z, p4[u].w};
          const uint32_t* r0 = &r[u][0].x;
          const uint32_t* r1 = &r[u][1].x;
          const uint32_t* r2 = &r[u][2].x;
          const uint32_t* r3 = &r[u][3].x;
          uint32_t o[4];
#pragma unroll
          for (int v = 0; v < 4; ++v) {
            float lo = p[0] * bf16_lo(r0[v]);
            lo = fmaf(p[1], bf16_lo(r1[v]), lo);
            lo = fmaf(p[2], bf16_lo(r2[v]), lo);
            lo = fmaf(p[3], bf16_lo(r3[v]), lo);
            float hi = p[0] * bf16_hi(r0[v]);
            hi = fmaf(p[1], bf16_hi(r1[v]), hi);
            hi = fmaf(p[2], bf16_hi(r2[v]), hi);
            hi = fmaf(p[3], bf16_hi(r3[v]), hi);
            o[v] = pack_bf16x2(lo, hi);
          }
          *reinterpret_cast<uint4*>(a.y + tok[u] * a.H + hc[u]) = make_uint4(o[0], o[1], o[2], o[3]);
        }
      }
    }
  }
  if (warp == kFuRelWarp && lane == 0) {
    // ---------------------------------------------------------------- count release
    int it = 0;
    for (int j = g; j < a.ntiles; j += a.groups, ++it) {
      const int rs = it & 1;
      if (!mbar_wait(&recdone[rs], static_cast<uint32_t>(it >> 1) & 1u, 37)) break;
      if (!status_set()) red_release_add(&a.cnt[j], 1);
      mbar_arrive(&recfree[rs]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kFuTmemCols)
                 : "memory");
  }
}

// Zeroes the tile counters; launched right before the fused kernel.
__global__ void pre_fused_zero_kernel(int* cnt, int n) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) cnt[i] = 0;
}

// 3-D bf16 tensor map over [d2][4][H] (H contiguous), box [box2][1][box0].
static bool make_map_3d(CUtensorMap* m, const void* base, int64_t H, int64_t d2, int box0,
                        int box2, CUtensorMapSwizzle swz) {
  EncodeTiledFn fn = encode_tiled();
  if (!fn) return false;
  const cuuint64_t dims[3] = {static_cast<cuuint64_t>(H), 4, static_cast<cuuint64_t>(d2)};
  const cuuint64_t strides[2] = {static_cast<cuuint64_t>(H) * 2, static_cast<cuuint64_t>(H) * 8};
  const cuuint32_t box[3] = {static_cast<cuuint32_t>(box0), 1, static_cast<cuuint32_t>(box2)};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, swz, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Returns 0, a negative MHC_ERR_* code, or 1 when this device cannot co-schedule the grid (the
// caller then takes another path).
int launch_pre_fused(const PreArgs& a, cudaStream_t s) {
  const FuPlan plan = fu_plan(a.T, a.H);
  const int sms = device_sm_count();
  if (plan.nsg > sms) return 1;
  int64_t groups = sms / plan.nsg;
  if (groups > plan.gmax) groups = plan.gmax;  // the workspace holds gmax record rings
  const int q = static_cast<int>(plan.q);
  const int smem = fu_smem_bytes(q);

  static bool attr_set[64] = {};
  const int dev = current_device();
  if (dev < 0) return -4;
  if (!attr_set[dev]) {
    const int mx = fu_smem_bytes(1) > fu_smem_bytes(2) ? fu_smem_bytes(1) : fu_smem_bytes(2);
    if (cudaFuncSetAttribute(pre_fused_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, mx) !=
        cudaSuccess)
      return -4;
    attr_set[dev] = true;
  }
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pre_fused_kernel, kFuThreads, smem) !=
          cudaSuccess ||
      per_sm < 1)
    return 1;

  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  uint16_t* Bw = reinterpret_cast<uint16_t*>(ws);
  int* cnt = reinterpret_cast<int*>(ws + plan.cnt_off);
  float* part = reinterpret_cast<float*>(ws + plan.part_off);
  CUtensorMap mR, mB;
  if (!make_map_3d(&mR, a.R, a.H, a.T, kFuHS, kFuM, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_3d(&mB, Bw, a.H, kFuN, kFuHS, kFuN, CU_TENSOR_MAP_SWIZZLE_128B))
    return -4;

  const int64_t K = 4 * a.H;
  const int64_t sb = (K + 255) / 256;
  pre_tc_split_kernel<<<static_cast<int>(sb < 4096 ? sb : 4096), 256, 0, s>>>(a.hc_fn, Bw, K);
  pre_fused_zero_kernel<<<1, 256, 0, s>>>(cnt, static_cast<int>(2 * plan.ntiles));
  note_launches(2);
  if (cudaGetLastError() != cudaSuccess) return -4;

  FuArgs fa;
  fa.R = a.R;
  fa.scale = a.hc_scale;
  fa.base = a.hc_base;
  fa.y = a.y;
  fa.pre = a.pre;
  fa.post = a.post;
  fa.comb = a.comb;
  fa.cnt = cnt;
  fa.ready = cnt + plan.ntiles;
  fa.part = part;
  fa.T = a.T;
  fa.H = a.H;
  fa.ntiles = static_cast<int>(plan.ntiles);
  fa.nsg = static_cast<int>(plan.nsg);
  fa.q = q;
  fa.groups = static_cast<int>(groups);
  fa.fp = FinishParams{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};

  void* args[] = {&mR, &mB, &fa};
  const dim3 grid(static_cast<unsigned>(plan.nsg * groups));
  if (cudaLaunchCooperativeKernel(reinterpret_cast<const void*>(pre_fused_kernel), grid,
                                  dim3(kFuThreads), args, static_cast<size_t>(smem), s) !=
      cudaSuccess)
    return -4;
  note_launches(1);
  return 0;
}

}  // namespace mhc
