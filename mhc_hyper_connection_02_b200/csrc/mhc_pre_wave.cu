// mHC pre-map in one pass over R, wavefront order: every CTA projects a short K range of the same
// few token tiles at a time, so each tile is complete soon after it was read, and the aggregate's
// re-read of its rows is served by L2 instead of HBM.
//
// Work layout. R is the flattened [T][4H] matrix (k = i*H + h) cut into 64-wide K blocks; the
// units (tile of 128 tokens, K block) are numbered tile-major and cut into ranges of RL
// consecutive units. Range r belongs to CTA r mod P (P CTAs, one per SM, cooperative launch), which
// takes its ranges in order; so at any moment the P CTAs work on neighbouring tiles, and tile t is
// finished once the ranges that overlap it are. A range is one or two pieces (it may cross a tile
// boundary); a piece is accumulated on tcgen05 into one TMEM accumulator (M=128, N=80: the exact
// bf16 x3 split of hc_fn [hi | mid | lo] as in mhc_pre_tc.cu, B tiles streamed from L2) and becomes
// the partial record rec[tile][row][slot] = raw[24], ss, where slot = the piece's rank among the
// tile's pieces. Inside a CTA:
//
//   warp 0      TMA: per K block one R tile [128 x 64] and one Bw tile [80 x 64] (128-byte swizzle)
//               into an 8-stage ring. Before a range whose first unit lies in tile t it waits until
//               this CTA's own aggregate units of tile t - D are done: that bounds how far the
//               stream runs ahead of the aggregate, hence how much of R must stay in L2.
//   warp 1      tcgen05.mma, K=16 steps, into two TMEM accumulators used by alternate pieces.
//   warps 2-5   sum of squares of each token row from the same stages; at the end of a piece the
//               accumulator (tcgen05.ld, eight columns at a time) and the record stores.
//   warp 6      publisher: one release-increment of the tile's piece counter per piece, once the
//               four record warps are done with it (its fence waits for their stores off the path
//               of the stage ring); then the accumulator goes back to the MMA warp.
//   warps 7-15  the aggregate, in units: per token `nparts` y units of at most 1024 columns and one
//               coefficient unit, numbered tile by tile and dealt to the CTAs in turn. A y unit
//               issues its row loads of R (an input, in L2 where the stream put it), then makes
//               sure the tile's records are published (a per-CTA note of the piece counters seen
//               complete, else the counter itself), sums the token's records in slot order (lane s
//               takes slots s and s + 32, then a fixed xor tree), forms rstd and the pre gates,
//               counts itself and writes its part of y = bf16_rn(sum_i pre_i R_i); the coefficient
//               unit writes pre, post and the comb logits instead. Units count in a per-CTA tally
//               per tile; the CTA's last unit of a tile adds the CTA's count to the tile's global
//               consumed counter with one release, and a record-ring slot (D + 10 tiles) is
//               rewritten only after that count is complete.
//
// A standalone Sinkhorn pass (mhc_sinkhorn.cu) then turns the comb logits into comb in place, and
// a one-grid prep kernel before the call splits hc_fn into Bw and zeroes the counters; the three
// are chained by programmatic dependent launch. Every wait is bounded by time: on expiry the kernel
// records MHC_ERR_TIMEOUT in the device status word and winds down (copies in flight drained,
// TMEM released after the last MMA; the four record warps agree on stopping through bar.red.or).
//
// "FlashInfer mHC module deep dive" §3.3 (split reduction of dot_mix / sqrsum), §3.4 (per-token
// phases: sum of squares and rstd, gates, softmax and Sinkhorn rounds, vec8 aggregate), §5.2;
// glm5next_mhc.rs glm_hc_pre (mix, then finish). The TMA, descriptor and MMA helpers and the
// tensor-map encoder are those of mhc_pre_tc.cu (same translation unit).
#include <cuda.h>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kWvM = 128;                              // tokens per tile (MMA M)
constexpr int kWvN = 80;                               // 3 x 24 split columns + 8 zero rows
constexpr int kWvKB = 64;                              // K per block
constexpr int kWvABytes = kWvM * kWvKB * 2;            // 16384
constexpr int kWvBBytes = kWvN * kWvKB * 2;            // 10240
constexpr int kWvStageBytes = kWvABytes + kWvBBytes;   // 26624 = 26 x 1024
constexpr int kWvStages = 8;
constexpr int kWvRec = 28;                             // floats per record: raw[24], ss, 3 zero
constexpr int kWvPubWarp = 6;
constexpr int kWvAggWarp0 = 7;
constexpr int kWvAggWarps = 9;
constexpr int kWvThreads = 32 * (kWvAggWarp0 + kWvAggWarps);
constexpr int kWvTmemCols = 256;                       // accumulators at columns 0 and 128
constexpr int kWvLag = 6;                              // D, in tiles
constexpr int kWvRing = kWvLag + 10;                   // record ring, in tiles
constexpr int kWvSub = 8;                              // consumed sub-counters per tile
constexpr int kWvMaxCtas = 148;
constexpr int kWvPartGroups = 128;                     // most 8-column groups in a y unit
constexpr int kWvMaxPieces = 33;                       // pieces of one tile at most (two per lane)
constexpr int kWvTSlots = 64;                         // per-tile words in shared memory
constexpr int kWvSmem = 1024 + kWvStages * kWvStageBytes + 256 + 3 * kWvTSlots * 4;
static_assert(kWvPartGroups == 4 * 32, "a y unit is at most four 8-column groups per lane");

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, uint32_t (&r)[8]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7])
      : "r"(taddr)
      : "memory");
}

struct WvPlan {
  bool ok;
  int64_t K, KB, ntiles, RL, nranges, Smax;
  int P, nparts;
  size_t cnt_off, cons_off, rec_off, total;
};

static WvPlan wv_plan(int64_t T, int64_t H, int sms) {
  WvPlan p{};
  p.ok = false;
  if (T < 1 || H < 64 || H % 8 != 0 || sms < 1) return p;
  p.P = sms < kWvMaxCtas ? sms : kWvMaxCtas;
  p.K = 4 * H;
  p.KB = (p.K + kWvKB - 1) / kWvKB;
  p.ntiles = (T + kWvM - 1) / kWvM;
  if (p.ntiles > (int64_t(1) << 24) || p.KB > (int64_t(1) << 24)) return p;
  // At most 32 ranges meet in a tile (33 pieces: records and their sums stay small), at least 4
  // blocks per range.
  p.RL = (p.KB + 31) / 32;
  if (p.RL < 4) p.RL = 4;
  p.nranges = (p.ntiles * p.KB + p.RL - 1) / p.RL;
  p.Smax = (p.KB + p.RL - 1) / p.RL + 1;
  if (p.Smax > kWvMaxPieces) return p;
  const int64_t H8 = H / 8;
  p.nparts = static_cast<int>((H8 + kWvPartGroups - 1) / kWvPartGroups);
  p.cnt_off = (static_cast<size_t>(kWvN) * p.K * 2 + 1023) / 1024 * 1024;  // after Bw
  p.cons_off = p.cnt_off + (static_cast<size_t>(p.ntiles) * 4 + 255) / 256 * 256;
  p.rec_off = p.cons_off + (static_cast<size_t>(p.ntiles) * kWvSub * 4 + 255) / 256 * 256;
  p.total = p.rec_off + static_cast<size_t>(kWvRing) * kWvM * p.Smax * kWvRec * 4;
  p.ok = true;
  return p;
}

bool pre_wave_supported(int64_t T, int64_t H) { return wv_plan(T, H, kWvMaxCtas).ok; }

size_t pre_wave_workspace_bytes(int64_t T, int64_t H) {
  const WvPlan p = wv_plan(T, H, kWvMaxCtas);
  return p.ok ? p.total : 0;
}

// ------------------------------------------------------------------------------ device helpers

// Waits until *p >= target (every lane polls; acquire). False on timeout or once another wait has
// timed out. The poll interval grows to 256 ns: many warps may wait on one counter.
__device__ __forceinline__ bool wv_wait_count(const int* p, int target, int where) {
  if (ld_acquire_gpu(p) >= target) return true;
  const unsigned long long t0 = global_timer_ns();
  unsigned ns = 32;
  for (uint32_t i = 1;; ++i) {
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
    if (ld_acquire_gpu(p) >= target) return true;
    if ((i & 15u) == 0) {
      if (*reinterpret_cast<volatile int*>(&g_device_status) != 0) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        report_timeout(where);
        return false;
      }
    }
  }
}

// Waits until the kWvSub sub-counters at p add up to at least target (acquire).
__device__ __forceinline__ bool wv_wait_sum(const int* p, int target, int where) {
  const unsigned long long t0 = global_timer_ns();
  unsigned ns = 32;
  for (uint32_t i = 0;; ++i) {
    int s = 0;
#pragma unroll
    for (int c = 0; c < kWvSub; ++c) s += ld_acquire_gpu(p + c);
    if (s >= target) return true;
    __nanosleep(ns);
    if (ns < 256) ns <<= 1;
    if ((i & 15u) == 15u) {
      if (*reinterpret_cast<volatile int*>(&g_device_status) != 0) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        report_timeout(where);
        return false;
      }
    }
  }
}

struct WvArgs {
  const uint16_t* R;
  const float* scale;
  const float* base;
  uint16_t* y;
  float* pre;
  float* post;
  float* comb;  // receives the comb logits; the Sinkhorn pass finishes it
  int* cnt;     // [ntiles] pieces published
  int* cons;    // [ntiles][kWvSub] aggregate units done
  float* rec;   // [kWvRing][128][Smax][kWvRec]
  int64_t T, H, K, KB, ntiles, RL, nranges;
  int Smax, nparts;
  float rms_eps, pre_eps, post_mult;
};

// Pieces that cover tile t (ranges r_first .. r_last) and the rank of range r among them.
__device__ __forceinline__ int64_t wv_first_range(int64_t t, int64_t KB, int64_t RL) {
  return t * KB / RL;
}
__device__ __forceinline__ int wv_pieces(int64_t t, int64_t KB, int64_t RL) {
  return static_cast<int>(((t + 1) * KB - 1) / RL - t * KB / RL + 1);
}
// Aggregate units of tile t: one coefficient unit and nparts y units per token.
__device__ __forceinline__ int wv_units(int64_t t, int64_t T, int nparts) {
  const int64_t n = T - t * kWvM;
  return static_cast<int>((n < kWvM ? n : kWvM) * (nparts + 1));
}

// Aggregate units of tile t that CTA j of P takes (unit numbers congruent to j modulo P).
__device__ __forceinline__ int wv_cta_units(int64_t t, int64_t per_tile, int nunits, int64_t j,
                                            int64_t P) {
  const int64_t a0 = t * per_tile;
  const int64_t first = a0 + ((j - a0) % P + P) % P;
  const int64_t end = a0 + nunits;
  return first >= end ? 0 : static_cast<int>((end - 1 - first) / P + 1);
}

__device__ __forceinline__ int ld_acquire_cta_shared(const int* p) {
  int v;
  asm volatile("ld.acquire.cta.shared::cta.b32 %0, [%1];" : "=r"(v) : "r"(smem_u32(p)) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_cta_shared(int* p, int v) {
  asm volatile("st.release.cta.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(p)), "r"(v) : "memory");
}

__device__ __forceinline__ int atom_add_acq_rel_cta_shared(int* p, int v) {
  int old;
  asm volatile("atom.acq_rel.cta.shared::cta.add.u32 %0, [%1], %2;"
               : "=r"(old)
               : "r"(smem_u32(p)), "r"(v)
               : "memory");
  return old;
}

// rstd and one pre gate, written once so that every unit of a token computes the same bits.
__device__ __forceinline__ float wv_rstd(float ss, float K, float rms_eps) {
  return __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(ss, K) + rms_eps));
}
__device__ __forceinline__ float wv_pre_gate(float raw, float rstd, float scale0, float base_r,
                                             float pre_eps) {
  return sigmoidf_ieee(fmaf(raw * rstd, scale0, base_r)) + pre_eps;
}

__global__ void __launch_bounds__(kWvThreads, 1)
    pre_wave_kernel(const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmB,
                    const WvArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + kWvStages * kWvStageBytes);
  uint64_t* empty = full + kWvStages;
  uint64_t* afull = empty + kWvStages;  // [2] accumulator b complete (MMA commit)
  uint64_t* aempty = afull + 2;         // [2] accumulator b read out and its records published
  uint64_t* recfull = aempty + 2;       // [2] piece records of accumulator b stored (4 warps)
  uint64_t* done = recfull + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  static_assert((2 * kWvStages + 7) * 8 + 4 <= 256, "barrier area");
  // Per-tile words, tile t in slot t % kWvTSlots (this CTA's stream and units all lie within a few
  // tens of tiles, fewer than kWvTSlots): units of the tile this CTA has finished; t + 1 once the
  // tile's records are known to be published; t + 1 once this CTA's units of the tile are done.
  int* tally = reinterpret_cast<int*>(smem + kWvStages * kWvStageBytes + 256);
  int* ready = tally + kWvTSlots;
  int* tdone = ready + kWvTSlots;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t j = blockIdx.x;
  const int64_t KB = a.KB, RL = a.RL;
  const int64_t units_total = a.ntiles * KB;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kWvStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA commit + one arrival per sum-of-squares warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], 1);   // the publisher
      mbar_init(&recfull[b], 4);  // one arrival per record warp
    }
    mbar_init(done, 1);
    for (int i = 0; i < 3 * kWvTSlots; ++i) tally[i] = 0;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kWvTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // Bw and the zeroed counters come from the prep grid launched just before

  const int64_t per_tile = static_cast<int64_t>(kWvM) * (a.nparts + 1);  // aggregate units
  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      for (int64_t r = j; r < a.nranges && ok; r += P) {
        const int64_t u0 = r * RL;
        const int64_t u1 = min(u0 + RL, units_total);
        const int64_t ts = u0 / KB;
        if (ts >= kWvLag) {
          // This CTA's own aggregate units of tile t - D are done (where it has any).
          const int64_t tw = ts - kWvLag;
          if (wv_cta_units(tw, per_tile, wv_units(tw, a.T, a.nparts), j, P) > 0) {
            const volatile int* td = tdone + (tw & (kWvTSlots - 1));
            const unsigned long long t0 = global_timer_ns();
            for (uint32_t i = 0; *td != static_cast<int>(tw) + 1; ++i) {
              __nanosleep(64);
              if ((i & 63u) == 63u) {
                if (*reinterpret_cast<volatile int*>(&g_device_status) != 0 ||
                    global_timer_ns() - t0 > kWaitLimitNs) {
                  report_timeout(70);
                  ok = false;
                  break;
                }
              }
            }
            if (!ok) break;
          }
        }
        for (int64_t u = u0; u < u1; ++u, ++it) {
          const int64_t tile = u / KB;
          const int kb = static_cast<int>(u - tile * KB);
          const int s = static_cast<int>(it % kWvStages);
          const uint32_t ph = static_cast<uint32_t>(it / kWvStages) & 1u;
          if (it >= kWvStages && !mbar_wait(&empty[s], ph ^ 1u, 71)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * kWvStageBytes;
          mbar_arrive_expect_tx(&full[s], kWvStageBytes);
          tma_load_2d(st, &tmR, kb * kWvKB, static_cast<int>(tile * kWvM), &full[s]);
          tma_load_2d(st + kWvABytes, &tmB, kb * kWvKB, 0, &full[s]);
        }
      }
      if (!ok) {  // do not leave while copies into shared memory are in flight
        for (int64_t i = it - kWvStages; i < it; ++i)
          if (i >= 0)
            mbar_wait(&full[i % kWvStages], static_cast<uint32_t>(i / kWvStages) & 1u, 72);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int64_t it = 0, pc = 0;
      bool ok = true;
      for (int64_t r = j; r < a.nranges && ok; r += P) {
        const int64_t u1 = min(r * RL + RL, units_total);
        for (int64_t u = r * RL; u < u1 && ok;) {
          const int64_t tile = u / KB;
          const int kbs = static_cast<int>(u - tile * KB);
          const int kbe = static_cast<int>(min(KB, kbs + (u1 - u)));
          const int b = static_cast<int>(pc & 1);
          if (pc >= 2 && !mbar_wait(&aempty[b], static_cast<uint32_t>((pc >> 1) - 1) & 1u, 73)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t dt = tmem + static_cast<uint32_t>(b * 128);
          for (int kb = kbs; kb < kbe; ++kb, ++it) {
            const int s = static_cast<int>(it % kWvStages);
            const uint32_t ph = static_cast<uint32_t>(it / kWvStages) & 1u;
            if (!mbar_wait(&full[s], ph, 74)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = smem_u32(smem + s * kWvStageBytes);
            const uint64_t adesc = sw128_desc(sa);
            const uint64_t bdesc = sw128_desc(sa + kWvABytes);
#pragma unroll
            for (int k = 0; k < kWvKB / 16; ++k)  // +32 bytes along the swizzled row per K=16 step
              umma_bf16(dt, adesc + 2 * k, bdesc + 2 * k, (kb > kbs || k > 0) ? 1u : 0u);
            umma_commit(&empty[s]);
          }
          if (!ok) break;
          umma_commit(&afull[b]);
          ++pc;
          u += kbe - kbs;
        }
      }
      // Every issued MMA has finished before TMEM is released.
      umma_commit(done);
      mbar_wait(done, 0, 75);
    }
  } else if (warp < kWvPubWarp) {
    // ------------------------------------------------------------------ sum of squares + records
    // TMEM lane quarter q = warp % 4 holds accumulator rows 32q .. 32q + 31; thread `row` also sums
    // the squares of token row `row` of each R tile.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int64_t it = 0, pc = 0;
    bool stop = false;
    for (int64_t r = j; r < a.nranges && !stop; r += P) {
      const int64_t u1 = min(r * RL + RL, units_total);
      for (int64_t u = r * RL; u < u1;) {
        const int64_t tile = u / KB;
        const int kbs = static_cast<int>(u - tile * KB);
        const int kbe = static_cast<int>(min(KB, kbs + (u1 - u)));
        bool ok = true;
        float ss0 = 0.f, ss1 = 0.f;
        for (int kb = kbs; kb < kbe; ++kb, ++it) {
          const int s = static_cast<int>(it % kWvStages);
          const uint32_t ph = static_cast<uint32_t>(it / kWvStages) & 1u;
          if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, 76))) {
            ok = false;
            break;
          }
          // Row `row` of the swizzled tile is its own 128 contiguous bytes (16-byte chunks permuted
          // within it); a sum does not depend on their order. Lanes start at different chunks.
          const uint4* rp = reinterpret_cast<const uint4*>(smem + s * kWvStageBytes + row * 128);
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 w = rp[cc ^ (lane & 7)];
            const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = bf16_lo(w4[e]), x1 = bf16_hi(w4[e]);
              ss0 = fmaf(x0, x0, ss0);
              ss1 = fmaf(x1, x1, ss1);
            }
          }
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[s]);
        }
        const int b = static_cast<int>(pc & 1);
        if (ok && !__all_sync(0xffffffffu,
                              mbar_wait(&afull[b], static_cast<uint32_t>(pc >> 1) & 1u, 77)))
          ok = false;
        // The record ring slot of this tile last held tile - kWvRing: every unit that read it has
        // finished (the stream's wait before this range already implies it; checked here too).
        if (ok && tile >= kWvRing) {
          const int64_t tw = tile - kWvRing;
          if (!__all_sync(0xffffffffu,
                          wv_wait_sum(a.cons + tw * kWvSub, wv_units(tw, a.T, a.nparts), 78)))
            ok = false;
        }
        if (ok) {
          tc_fence_after();
          const uint32_t tbase =
              tmem + static_cast<uint32_t>(b * 128) + (static_cast<uint32_t>(q * 32) << 16);
          const int64_t t = tile * kWvM + row;
          const int64_t slot = r - wv_first_range(tile, KB, RL);
          float4* r4 = reinterpret_cast<float4*>(
              a.rec +
              ((static_cast<size_t>(tile % kWvRing) * kWvM + row) * a.Smax + slot) * kWvRec);
          // Outputs 8g .. 8g + 7: their hi, mid and lo columns, eight at a time (few registers).
#pragma unroll
          for (int g = 0; g < 3; ++g) {
            uint32_t dh[8], dm[8], dl[8];
            tmem_ld8(tbase + 8 * g, dh);
            tmem_ld8(tbase + kMix + 8 * g, dm);
            tmem_ld8(tbase + 2 * kMix + 8 * g, dl);
            tmem_wait_ld();
            float v[8];
#pragma unroll
            for (int e = 0; e < 8; ++e)
              v[e] = (__uint_as_float(dl[e]) + __uint_as_float(dm[e])) + __uint_as_float(dh[e]);
            if (t < a.T) {
              r4[2 * g] = make_float4(v[0], v[1], v[2], v[3]);
              r4[2 * g + 1] = make_float4(v[4], v[5], v[6], v[7]);
            }
          }
          if (t < a.T) r4[6] = make_float4(ss0 + ss1, 0.f, 0.f, 0.f);
          // TMEM reads and record stores are done: the publisher takes it from here.
          tc_fence_before();
          __syncwarp();
          if (lane == 0) mbar_arrive(&recfull[b]);
        }
        ++pc;
        if (!ok) {
          stop = true;
          break;
        }
        u += kbe - kbs;
      }
    }
  } else if (warp == kWvPubWarp) {
    // ------------------------------------------------------------------ piece publisher
    // Once the four record warps have stored a piece's records, one release-increment of the
    // tile's piece counter publishes them (the gpu-scope fence covers the stores this thread
    // observed through the barrier); then the accumulator is free for the MMA. The fence's wait
    // for the stores to reach L2 stalls only this warp, not the stage ring.
    if (lane == 0) {
      int64_t pc = 0;
      bool ok = true;
      for (int64_t r = j; r < a.nranges && ok; r += P) {
        const int64_t u1 = min(r * RL + RL, units_total);
        for (int64_t u = r * RL; u < u1;) {
          const int64_t tile = u / KB;
          const int kbs = static_cast<int>(u - tile * KB);
          const int kbe = static_cast<int>(min(KB, kbs + (u1 - u)));
          const int b = static_cast<int>(pc & 1);
          if (!mbar_wait(&recfull[b], static_cast<uint32_t>(pc >> 1) & 1u, 80)) {
            ok = false;
            break;
          }
          red_release_add_gpu(a.cnt + tile, 1);
          mbar_arrive(&aempty[b]);
          ++pc;
          u += kbe - kbs;
        }
      }
    }
  } else {
    // ------------------------------------------------------------------ aggregate units
    const int wb = warp - kWvAggWarp0;
    const int upt = a.nparts + 1;
    const int64_t total = a.ntiles * per_tile;
    const int64_t H = a.H, H8 = H / 8;
    const int64_t gpp = (H8 + a.nparts - 1) / a.nparts;  // 8-column groups per y unit
    const float Kf = static_cast<float>(a.K);
    const float scale0 = __ldg(a.scale), scale1 = __ldg(a.scale + 1), scale2 = __ldg(a.scale + 2);
    // A finished unit adds one to this CTA's tally of its tile (acquire-release at CTA scope, so
    // the last one has seen every earlier unit's reads); the CTA's last unit of the tile resets the
    // slot and publishes the tile's count with one gpu-scope release-increment.
    auto count_unit = [&](int64_t t) {
      __syncwarp();
      if (lane == 0) {
        int* c = tally + (t & (kWvTSlots - 1));
        const int n = wv_cta_units(t, per_tile, wv_units(t, a.T, a.nparts), j, P);
        if (atom_add_acq_rel_cta_shared(c, 1) + 1 == n) {
          atomicExch(c, 0);
          red_release_add_gpu(a.cons + t * kWvSub + (j & (kWvSub - 1)), n);
          atomicExch(tdone + (t & (kWvTSlots - 1)), static_cast<int>(t) + 1);
        }
      }
    };
    // The tile's records are published: known to this CTA already (another warp saw the piece
    // counter complete), else wait for the counter and note it for the other warps.
    auto tile_ready = [&](int64_t t, int S) -> bool {
      int* rs = ready + (t & (kWvTSlots - 1));
      if (ld_acquire_cta_shared(rs) == static_cast<int>(t) + 1) return true;
      if (!__all_sync(0xffffffffu, wv_wait_count(a.cnt + t, S, 79))) return false;
      if (lane == 0) st_release_cta_shared(rs, static_cast<int>(t) + 1);
      return true;
    };
    for (int64_t m = wb;; m += kWvAggWarps) {
      const int64_t U = j + P * m;
      if (U >= total) break;
      const int64_t t = U / per_tile;
      const int v = static_cast<int>(U - t * per_tile);
      const int l = v / upt;
      const int part = v - l * upt;
      const int64_t tok = t * kWvM + l;
      if (tok >= a.T) continue;
      const int S = wv_pieces(t, KB, RL);
      const float* rt =
          a.rec + (static_cast<size_t>(t % kWvRing) * kWvM + l) * a.Smax * kWvRec;
      // S <= 33 pieces: lane s holds slots s and s + 32; the sums run (0 + first) + second, the
      // same association in both kinds of unit, so every unit of a token forms the same bits.
      const bool one = lane < S;
      const bool two = lane + 32 < S;
      if (part < a.nparts) {
        // y unit: this token's columns [g0, g1) x 8 of the four streams. R is an input: its
        // loads go out before the wait for the tile's records (they hit L2, where the stream put
        // the tile).
        const int64_t g0 = part * gpp;
        const int64_t g1 = min(g0 + gpp, H8);
        const uint16_t* rrow = a.R + tok * 4 * H;
        uint4 rv[4][4];
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t g = g0 + lane + 32 * i;
          if (g < g1) {
#pragma unroll
            for (int st = 0; st < 4; ++st) rv[i][st] = ld_stream_ro(rrow + st * H + g * 8);
          }
        }
        if (!tile_ready(t, S)) break;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        float4 a0 = z4, a6 = z4, b0 = z4, b6 = z4;
        if (one) {
          a0 = __ldcg(reinterpret_cast<const float4*>(rt + lane * kWvRec));
          a6 = __ldcg(reinterpret_cast<const float4*>(rt + lane * kWvRec + 24));
        }
        if (two) {
          b0 = __ldcg(reinterpret_cast<const float4*>(rt + (lane + 32) * kWvRec));
          b6 = __ldcg(reinterpret_cast<const float4*>(rt + (lane + 32) * kWvRec + 24));
        }
        float s0 = (0.f + a0.x) + b0.x, s1 = (0.f + a0.y) + b0.y, s2 = (0.f + a0.z) + b0.z;
        float s3 = (0.f + a0.w) + b0.w, sq = (0.f + a6.x) + b6.x;
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) {
          s0 += __shfl_xor_sync(0xffffffffu, s0, sh);
          s1 += __shfl_xor_sync(0xffffffffu, s1, sh);
          s2 += __shfl_xor_sync(0xffffffffu, s2, sh);
          s3 += __shfl_xor_sync(0xffffffffu, s3, sh);
          sq += __shfl_xor_sync(0xffffffffu, sq, sh);
        }
        const float rstd = wv_rstd(sq, Kf, a.rms_eps);
        const float p0 = wv_pre_gate(s0, rstd, scale0, __ldg(a.base), a.pre_eps);
        const float p1 = wv_pre_gate(s1, rstd, scale0, __ldg(a.base + 1), a.pre_eps);
        const float p2 = wv_pre_gate(s2, rstd, scale0, __ldg(a.base + 2), a.pre_eps);
        const float p3 = wv_pre_gate(s3, rstd, scale0, __ldg(a.base + 3), a.pre_eps);
        // The unit's record reads are done: count it now, before its y stores.
        count_unit(t);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          const int64_t g = g0 + lane + 32 * i;
          if (g < g1) {
            const uint32_t* r0 = &rv[i][0].x;
            const uint32_t* r1 = &rv[i][1].x;
            const uint32_t* r2 = &rv[i][2].x;
            const uint32_t* r3 = &rv[i][3].x;
            uint32_t o[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float lo = p0 * bf16_lo(r0[c]);
              lo = fmaf(p1, bf16_lo(r1[c]), lo);
              lo = fmaf(p2, bf16_lo(r2[c]), lo);
              lo = fmaf(p3, bf16_lo(r3[c]), lo);
              float hi = p0 * bf16_hi(r0[c]);
              hi = fmaf(p1, bf16_hi(r1[c]), hi);
              hi = fmaf(p2, bf16_hi(r2[c]), hi);
              hi = fmaf(p3, bf16_hi(r3[c]), hi);
              o[c] = pack_bf16x2(lo, hi);
            }
            st_stream(a.y + tok * H + g * 8, make_uint4(o[0], o[1], o[2], o[3]));
          }
        }
      } else {
        // Coefficient unit: all 25 sums, then lane q < 4 writes pre q, post q and comb row q.
        if (!tile_ready(t, S)) break;
        float acc[25];
        {
          const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
          float4 va[7], vb[7];
#pragma unroll
          for (int w = 0; w < 7; ++w) {
            va[w] = one ? __ldcg(reinterpret_cast<const float4*>(rt + lane * kWvRec) + w) : z4;
            vb[w] = two ? __ldcg(reinterpret_cast<const float4*>(rt + (lane + 32) * kWvRec) + w)
                        : z4;
          }
#pragma unroll
          for (int w = 0; w < 6; ++w) {
            acc[4 * w] = (0.f + va[w].x) + vb[w].x;
            acc[4 * w + 1] = (0.f + va[w].y) + vb[w].y;
            acc[4 * w + 2] = (0.f + va[w].z) + vb[w].z;
            acc[4 * w + 3] = (0.f + va[w].w) + vb[w].w;
          }
          acc[24] = (0.f + va[6].x) + vb[6].x;
        }
#pragma unroll
        for (int sh = 16; sh >= 1; sh >>= 1) {
#pragma unroll
          for (int c = 0; c < 25; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], sh);
        }
        if (lane < 4) {
          const int q = lane;
          const float rstd = wv_rstd(acc[24], Kf, a.rms_eps);
          const float g0 = q == 0 ? acc[0] : q == 1 ? acc[1] : q == 2 ? acc[2] : acc[3];
          const float g1 = q == 0 ? acc[4] : q == 1 ? acc[5] : q == 2 ? acc[6] : acc[7];
          a.pre[tok * 4 + q] = wv_pre_gate(g0, rstd, scale0, __ldg(a.base + q), a.pre_eps);
          a.post[tok * 4 + q] =
              a.post_mult * sigmoidf_ieee(fmaf(g1 * rstd, scale1, __ldg(a.base + 4 + q)));
          float cr[4];
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const float gc = q == 0   ? acc[8 + c]
                             : q == 1 ? acc[12 + c]
                             : q == 2 ? acc[16 + c]
                                      : acc[20 + c];
            cr[c] = fmaf(gc * rstd, scale2, __ldg(a.base + 8 + 4 * q + c));
          }
          *reinterpret_cast<float4*>(a.comb + tok * 16 + 4 * q) =
              make_float4(cr[0], cr[1], cr[2], cr[3]);
        }
        // The unit's reads of the tile's records are done (the ring slot may be reused once all
        // of the tile's units have counted).
        count_unit(t);
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kWvTmemCols)
                 : "memory");
  }
}

// Splits hc_fn into Bw (as pre_tc_split_kernel) and zeroes the wave counters; one grid before the
// wave kernel.
__global__ void __launch_bounds__(256) pre_wave_prep_kernel(const float* __restrict__ W,
                                                            uint16_t* __restrict__ Bw, int64_t K,
                                                            int* __restrict__ counters,
                                                            int64_t ncounters) {
  pdl_wait();  // the previous call's kernels may still read Bw or the counters
  pdl_trigger();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t i0 = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  for (int64_t k = i0; k < K; k += stride) split_hc_fn_row(W, Bw, K, k);
  for (int64_t i = i0; i < ncounters; i += stride) counters[i] = 0;
}

// ------------------------------------------------------------------------------ host side

// Returns 0, a negative MHC_ERR_* code, or 1 when this device cannot run the plan's grid with every
// CTA resident (nothing is launched then).
int launch_pre_wave(const PreArgs& a, cudaStream_t s) {
  const WvPlan plan = wv_plan(a.T, a.H, device_sm_count());
  if (!plan.ok) return 1;
  if (!ensure_smem_limit(reinterpret_cast<const void*>(pre_wave_kernel), kWvSmem)) return 1;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pre_wave_kernel, kWvThreads,
                                                    kWvSmem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return 1;
  }
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  uint16_t* Bw = reinterpret_cast<uint16_t*>(ws);
  int* cnt = reinterpret_cast<int*>(ws + plan.cnt_off);
  int* cons = reinterpret_cast<int*>(ws + plan.cons_off);
  float* rec = reinterpret_cast<float*>(ws + plan.rec_off);

  CUtensorMap mR, mB;
  if (!make_map(&mR, a.R, plan.K, a.T, kWvM) || !make_map(&mB, Bw, plan.K, kWvN, kWvN)) return -4;

  const int64_t sb = (plan.K + 255) / 256;
  const int prep_blocks = static_cast<int>(sb < 4096 ? sb : 4096);
  const int64_t ncounters = static_cast<int64_t>((plan.rec_off - plan.cnt_off) / 4);
  if (launch_pdl(pre_wave_prep_kernel, dim3(prep_blocks), dim3(256), 0, s,
                 static_cast<const float*>(a.hc_fn), Bw, plan.K, cnt, ncounters) != cudaSuccess)
    return -4;
  note_launches(1);

  WvArgs wa;
  wa.R = a.R;
  wa.scale = a.hc_scale;
  wa.base = a.hc_base;
  wa.y = a.y;
  wa.pre = a.pre;
  wa.post = a.post;
  wa.comb = a.comb;
  wa.cnt = cnt;
  wa.cons = cons;
  wa.rec = rec;
  wa.T = a.T;
  wa.H = a.H;
  wa.K = plan.K;
  wa.KB = plan.KB;
  wa.ntiles = plan.ntiles;
  wa.RL = plan.RL;
  wa.nranges = plan.nranges;
  wa.Smax = static_cast<int>(plan.Smax);
  wa.nparts = plan.nparts;
  wa.rms_eps = a.rms_eps;
  wa.pre_eps = a.pre_eps;
  wa.post_mult = a.post_mult;

  // Cooperative launch: every CTA resident at once (CTAs wait on one another's counters). Also a
  // programmatic dependent of the prep grid where the runtime accepts both attributes together.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.P));
  cfg.blockDim = dim3(kWvThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(kWvSmem);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, pre_wave_kernel, mR, mB, wa);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, pre_wave_kernel, mR, mB, wa);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return -4;
  }
  note_launches(1);
  // comb holds the logits: the Sinkhorn rounds run in place.
  return launch_sinkhorn(a.comb, a.comb, a.T, a.iters, a.sinkhorn_eps, s);
}

}  // namespace mhc
