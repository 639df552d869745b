// mHC pre-map in one pass over R: a persistent kernel that projects each token tile on tcgen05
// tensor cores, reduces the split partials across the CTAs of a group, forms the coefficients and
// aggregates y while the tile is still in L2.
//
// Work layout. R is the flattened [T][4H] matrix (k = i*H + h) cut into 64-wide K blocks. The
// launch is NG groups of G CTAs (NG * G <= SM count, one CTA per SM, cooperative launch so that all
// of them are resident together). CTA j of a group owns a fixed, contiguous range of K blocks (the
// ranges of a group cover K once) and keeps that slice of hc_fn resident in shared memory for the
// whole call as the MMA B operand: each weight split exactly into three bf16 terms hi + mid + lo
// (B rows [hi 24 | mid 24 | lo 24 | 8 zero], 128-byte swizzle, as in mhc_pre_tc.cu). Group g takes
// the token tiles (128 tokens) g, g + NG, g + 2 NG, ... in that order, and every CTA of the group
// projects its K range of each of them. Per tile n of a group, inside a CTA:
//
//   warp 0      TMA: one [128 x 64] R block per stage of a ring (128-byte swizzle). Before tile n
//               it waits until this CTA's coefficients of tile n - D are done: that bounds how far
//               the stream runs ahead of the aggregate, and so how much of R must stay in L2.
//   warp 1      tcgen05.mma M=128 N=80 K=16 over the K range into one of two TMEM accumulators.
//   warps 2-5   sum of squares of each token row from the same stages; after the tile, the
//               accumulator (tcgen05.ld) gives the partial record rec[token][j] = raw[24], ss, and
//               one thread release-increments the tile's counter.
//   warps 6-7   (tile n by warp 6 + n mod 2) once the counter reaches G: for the tokens this CTA
//               owns in the tile (token l with (l + 128 n) mod G == j), two at a time, sixteen
//               lanes per token sum its G partial records in a fixed order; then rstd, the logits,
//               the gates and the Sinkhorn comb; write pre, post and comb, and hand pre to the
//               aggregate warps through shared memory.
//   warps 8-15  y = bf16_rn(sum_i pre_i R_i) for the owned tokens, re-reading their rows with
//               16-byte loads. The tile came from HBM a few microseconds earlier and is still in
//               L2, so HBM sees R once.
//
// The tile counters are zeroed by a one-block kernel launched just before (programmatic dependent
// launch). Every wait is bounded by time: on expiry the kernel records MHC_ERR_TIMEOUT in the device
// status word and winds down (copies in flight are drained, TMEM is released after the last MMA).
//
// "FlashInfer mHC module deep dive" §3.3 (split reduction of dot_mix / sqrsum), §3.4 (per-token
// phases: sum of squares and rstd, gates, softmax and Sinkhorn rounds, vec8 aggregate), §5.2;
// glm5next_mhc.rs glm_hc_pre (mix, then finish).
#include <cuda.h>

#include <mutex>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kFsM = 128;                    // tokens per tile (MMA M)
constexpr int kFsN = 80;                     // 3 x 24 split columns + 8 zero rows
constexpr int kFsKB = 64;                    // K per block: one 128-byte swizzled row
constexpr int kFsABytes = kFsM * kFsKB * 2;  // 16384: one R block
constexpr int kFsBBytes = kFsN * kFsKB * 2;  // 10240: one resident hc_fn block
constexpr int kFsMaxNb = 13;                 // most resident K blocks per CTA
constexpr int kFsMinG = 4;                   // fewest CTAs per group
constexpr int kFsMaxOwn = kFsM / kFsMinG;    // most tokens a CTA owns in one tile
constexpr int kFsMaxStages = 8;
constexpr int kFsRec = 28;                   // floats per partial record (raw[24], ss, 3 zero)
constexpr int kFsEpiDelay = 3;              // stages into the next tile before the records
constexpr int kFsCoefWarps = 2;
constexpr int kFsTokLanes = 16;              // lanes that reduce one token's records
constexpr int kFsTokPerPass = 32 / kFsTokLanes;
constexpr int kFsSlots = 8;                  // coefficient -> aggregate hand-over slots
constexpr int kFsCoefWarp0 = 6;
constexpr int kFsAggWarp0 = kFsCoefWarp0 + kFsCoefWarps;
constexpr int kFsAggWarps = 8;
constexpr int kFsThreads = 32 * (kFsAggWarp0 + kFsAggWarps);
constexpr int kFsTmemCols = 256;             // accumulators at columns 0 and 128
constexpr int kFsMaxCtas = 148;              // most CTAs a plan uses (workspace sizing)
constexpr int kFsSmemLimit = 227 * 1024;
// D: the stream of tile n waits for this CTA's coefficients of tile n - D. D < kFsSlots keeps that
// wait unambiguous (the slot cannot have moved on by two phases), and a record ring of 2 D tiles
// is then never overwritten before every CTA of the group has read it.
constexpr int kFsLag = 4;
constexpr int kFsRing = 2 * kFsLag;
static_assert(kFsLag < kFsSlots, "lag must stay below the hand-over slots");

// Shared-memory scratch after the rings: barriers, TMEM address, coefficient sums, hand-over.
constexpr int kFsOffBars = 0;  // full[8] empty[8] afull[2] aempty[2] cfull[slots] cempty[slots] done
constexpr int kFsOffTmem = (2 * kFsMaxStages + 4 + 2 * kFsSlots + 1) * 8;
constexpr int kFsOffPre = (kFsOffTmem + 4 + 127) / 128 * 128;          // float [slots][own][4]
constexpr int kFsOffTok = kFsOffPre + kFsSlots * kFsMaxOwn * 16;       // int [slots][own]
constexpr int kFsOffNown = kFsOffTok + kFsSlots * kFsMaxOwn * 4;       // int [slots]
constexpr int kFsMisc = (kFsOffNown + kFsSlots * 4 + 127) / 128 * 128;

struct FsPlan {
  bool ok;
  int64_t KB;      // K blocks
  int64_t ntiles;  // token tiles
  int G, NG;       // CTAs per group, groups
  int nbmax;       // most K blocks of a CTA
  int stages;      // R ring depth
  int smem;        // dynamic shared memory bytes
  size_t cnt_off, rec_off, total;
};

static FsPlan fs_plan(int64_t T, int64_t H, int sms) {
  FsPlan p{};
  p.ok = false;
  if (T < 1 || H < 8 || H % 8 != 0 || sms < kFsMinG) return p;
  if (sms > kFsMaxCtas) sms = kFsMaxCtas;
  const int64_t K = 4 * H;
  p.KB = (K + kFsKB - 1) / kFsKB;
  p.ntiles = (T + kFsM - 1) / kFsM;
  if (p.ntiles > (int64_t(1) << 30)) return p;
  int64_t G = (p.KB + kFsMaxNb - 1) / kFsMaxNb;
  if (G < kFsMinG) G = kFsMinG;
  if (G > sms || G > p.KB) return p;
  int64_t NG = sms / G;
  if (NG > p.ntiles) NG = p.ntiles;
  G = sms / NG;  // spread the groups over every SM
  if (G > p.KB) G = p.KB;
  p.G = static_cast<int>(G);
  p.NG = static_cast<int>(NG);
  p.nbmax = static_cast<int>((p.KB + G - 1) / G);
  if (p.nbmax > kFsMaxNb) return p;
  const int fixed = 1024 + p.nbmax * kFsBBytes + kFsMisc;
  int st = (kFsSmemLimit - fixed) / kFsABytes;
  if (st > kFsMaxStages) st = kFsMaxStages;
  if (st < 2) return p;
  p.stages = st;
  p.smem = fixed + st * kFsABytes;
  p.cnt_off = 0;
  p.rec_off = (static_cast<size_t>(p.ntiles) * 4 + 255) / 256 * 256;
  p.total = p.rec_off + static_cast<size_t>(p.NG) * kFsRing * kFsM * p.G * kFsRec * 4;
  p.ok = true;
  return p;
}

bool pre_fused_supported(int64_t T, int64_t H) { return fs_plan(T, H, kFsMaxCtas).ok; }

// Where the single pass is the faster of the two tensor-core forms (measured on B200, device time):
// a few tiles per group (T up to ~1.5k tokens) and groups wide enough that each CTA owns at most
// 8 tokens of a tile. T=256..1024 at H=4096/7168: 24-50 us against 32-69 us for the split chain;
// from T=2048 (H=4096) and T=3072 (H=7168), or with narrow groups (H=1000), the split chain wins.
bool pre_fused_preferred(int64_t T, int64_t H) {
  const FsPlan p = fs_plan(T, H, kFsMaxCtas);
  return p.ok && T <= 1536 && p.G >= 16;
}

size_t pre_fused_workspace_bytes(int64_t T, int64_t H) {
  // The largest plan: records for every CTA of a full-size launch. Plans on devices with fewer SMs
  // need no more.
  const FsPlan p = fs_plan(T, H, kFsMaxCtas);
  if (!p.ok) return 0;
  return p.rec_off + static_cast<size_t>(kFsMaxCtas) * kFsRing * kFsM * kFsRec * 4;
}

// ------------------------------------------------------------------------------ device helpers

__device__ __forceinline__ void fs_tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                               uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fs_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void fs_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor: K-major, 128-byte swizzle, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t fs_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

// Instruction descriptor, kind::f16: D fp32, A and B bf16, both K-major, M = 128, N = 80.
constexpr uint32_t kFsIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kFsN >> 3) << 17) |
                              (static_cast<uint32_t>(kFsM >> 4) << 24);

__device__ __forceinline__ void fs_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                       uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kFsIdesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ void fs_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

__device__ __forceinline__ void fs_tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
}

// Waits until *p >= target (acquire); false on timeout or once another wait has timed out.
__device__ __noinline__ bool fs_wait_count(const int* p, int target, int where) {
  if (ld_acquire_gpu(p) >= target) return true;
  const unsigned long long t0 = global_timer_ns();
  for (uint32_t i = 1;; ++i) {
    __nanosleep(32);
    if (ld_acquire_gpu(p) >= target) return true;
    if ((i & 63u) == 0) {
      if (*reinterpret_cast<volatile int*>(&g_device_status) != 0) return false;
      if (global_timer_ns() - t0 > kWaitLimitNs) {
        report_timeout(where);
        return false;
      }
    }
  }
}

// Streaming read of data this kernel does not write; L1 not allocated.
__device__ __forceinline__ uint4 fs_ld_ro(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

struct FsArgs {
  const uint16_t* R;
  const float* hc_fn;
  const float* scale;
  const float* base;
  uint16_t* y;
  float* pre;
  float* post;
  float* comb;
  int* cnt;    // [ntiles]
  float* rec;  // [NG][kFsRing][128][G][kFsRec]
  int64_t T, H, K;
  int KB, ntiles, G, NG, nbmax, stages, lag;
  FinishParams fp;
};

__global__ void __launch_bounds__(kFsThreads, 1)
    pre_fused_kernel(const __grid_constant__ CUtensorMap tmR, const FsArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* Bres = smem;                                       // nbmax resident hc_fn blocks
  uint8_t* Aring = smem + a.nbmax * kFsBBytes;                // R ring
  uint8_t* misc = Aring + a.stages * kFsABytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(misc + kFsOffBars);
  uint64_t* empty = full + kFsMaxStages;
  uint64_t* afull = empty + kFsMaxStages;
  uint64_t* aempty = afull + 2;
  uint64_t* cfull = aempty + 2;
  uint64_t* cempty = cfull + kFsSlots;
  uint64_t* done = cempty + kFsSlots;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(misc + kFsOffTmem);
  float* slot_pre = reinterpret_cast<float*>(misc + kFsOffPre);
  int* slot_tok = reinterpret_cast<int*>(misc + kFsOffTok);
  int* slot_nown = reinterpret_cast<int*>(misc + kFsOffNown);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int G = a.G, NG = a.NG, ST = a.stages;
  const int g = blockIdx.x / G;
  const int j = blockIdx.x - g * G;
  const int kb0 = static_cast<int>(static_cast<int64_t>(j) * a.KB / G);
  const int nb = static_cast<int>(static_cast<int64_t>(j + 1) * a.KB / G) - kb0;
  const int ntg = (a.ntiles - g + NG - 1) / NG;  // tiles of this group

  if (threadIdx.x == 0) {
    for (int s = 0; s < kFsMaxStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA commit + one arrival per sum-of-squares warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], 4);
    }
    for (int s = 0; s < kFsSlots; ++s) {
      mbar_init(&cfull[s], 1);
      mbar_init(&cempty[s], kFsAggWarps);
    }
    mbar_init(done, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kFsTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  pdl_wait();  // the counters were zeroed by the grid launched just before
  pdl_trigger();

  // Resident B operand: hc_fn rows [kb0 * 64, (kb0 + nb) * 64) split into three exact bf16 terms.
  // Tile b holds rows r = 0..79 of 128 bytes; the 16-byte chunk c (k = 8c .. 8c + 7) of row r sits
  // at chunk position c ^ (r & 7) (the 128-byte swizzle the MMA descriptor names).
  {
    const int items = nb * 8 * kMix;
    for (int i = threadIdx.x; i < items; i += kFsThreads) {
      const int col = i % kMix;
      const int rest = i / kMix;
      const int c = rest & 7;
      const int b = rest >> 3;
      const int64_t k0 = static_cast<int64_t>(kb0 + b) * kFsKB + c * 8;
      uint32_t hi[4], mid[4], lo[4];
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        uint16_t h2[2], m2[2], l2[2];
#pragma unroll
        for (int u = 0; u < 2; ++u) {
          const int64_t k = k0 + e + u;
          const float w = k < a.K ? __ldg(a.hc_fn + k * kMix + col) : 0.f;
          h2[u] = f32_to_bf16(w);
          const float r1 = w - bf16_to_f32(h2[u]);
          m2[u] = f32_to_bf16(r1);
          const float r2 = r1 - bf16_to_f32(m2[u]);
          l2[u] = f32_to_bf16(r2);
        }
        hi[e / 2] = static_cast<uint32_t>(h2[0]) | (static_cast<uint32_t>(h2[1]) << 16);
        mid[e / 2] = static_cast<uint32_t>(m2[0]) | (static_cast<uint32_t>(m2[1]) << 16);
        lo[e / 2] = static_cast<uint32_t>(l2[0]) | (static_cast<uint32_t>(l2[1]) << 16);
      }
      uint8_t* tile = Bres + b * kFsBBytes;
      const int r0 = col, r1 = kMix + col, r2 = 2 * kMix + col;
      *reinterpret_cast<uint4*>(tile + r0 * 128 + ((c ^ (r0 & 7)) << 4)) =
          make_uint4(hi[0], hi[1], hi[2], hi[3]);
      *reinterpret_cast<uint4*>(tile + r1 * 128 + ((c ^ (r1 & 7)) << 4)) =
          make_uint4(mid[0], mid[1], mid[2], mid[3]);
      *reinterpret_cast<uint4*>(tile + r2 * 128 + ((c ^ (r2 & 7)) << 4)) =
          make_uint4(lo[0], lo[1], lo[2], lo[3]);
    }
    for (int i = threadIdx.x; i < nb * 8 * 8; i += kFsThreads) {  // rows 72..79: zero
      const int b = i >> 6;
      const int r = 3 * kMix + ((i >> 3) & 7);
      *reinterpret_cast<uint4*>(Bres + b * kFsBBytes + r * 128 + ((i & 7) << 4)) =
          make_uint4(0u, 0u, 0u, 0u);
    }
    // Generic-proxy writes become visible to the tensor cores' (async proxy) reads.
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  fs_fence_before();
  __syncthreads();
  fs_fence_after();
  const uint32_t tmem = *tmem_slot;
  float* const rec_g = a.rec + static_cast<size_t>(g) * kFsRing * kFsM * G * kFsRec;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      for (int n = 0; n < ntg && ok; ++n) {
        if (n >= a.lag) {
          const int m = n - a.lag;
          if (!mbar_wait(&cfull[m % kFsSlots], static_cast<uint32_t>(m / kFsSlots) & 1u, 40)) {
            ok = false;
            break;
          }
        }
        const int X = g + n * NG;
        for (int b = 0; b < nb; ++b, ++it) {
          const int s = static_cast<int>(it % ST);
          const uint32_t ph = static_cast<uint32_t>(it / ST) & 1u;
          if (it >= ST && !mbar_wait(&empty[s], ph ^ 1u, 41)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&full[s], kFsABytes);
          fs_tma_load_2d(Aring + s * kFsABytes, &tmR, (kb0 + b) * kFsKB, X * kFsM, &full[s]);
        }
      }
      if (!ok) {  // do not leave while copies into shared memory are in flight
        for (int64_t i = it - ST; i < it; ++i)
          if (i >= 0) mbar_wait(&full[i % ST], static_cast<uint32_t>(i / ST) & 1u, 42);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      for (int n = 0; n < ntg && ok; ++n) {
        const int b = n & 1;
        if (n >= 2 && !mbar_wait(&aempty[b], static_cast<uint32_t>((n >> 1) - 1) & 1u, 43)) {
          ok = false;
          break;
        }
        fs_fence_after();
        const uint32_t dt = tmem + static_cast<uint32_t>(b * 128);
        for (int kb = 0; kb < nb; ++kb, ++it) {
          const int s = static_cast<int>(it % ST);
          const uint32_t ph = static_cast<uint32_t>(it / ST) & 1u;
          if (!mbar_wait(&full[s], ph, 44)) {
            ok = false;
            break;
          }
          fs_fence_after();
          const uint64_t adesc = fs_desc(smem_u32(Aring + s * kFsABytes));
          const uint64_t bdesc = fs_desc(smem_u32(Bres + kb * kFsBBytes));
#pragma unroll
          for (int k = 0; k < kFsKB / 16; ++k)  // +32 bytes along the swizzled row per K=16 step
            fs_mma(dt, adesc + 2 * k, bdesc + 2 * k, (kb > 0 || k > 0) ? 1u : 0u);
          fs_commit(&empty[s]);
        }
        if (!ok) break;
        fs_commit(&afull[b]);
      }
      // Every issued MMA has finished before TMEM is released.
      fs_commit(done);
      mbar_wait(done, 0, 45);
    }
  } else if (warp < kFsCoefWarp0) {
    // ------------------------------------------------------------------ sum of squares + records
    // TMEM lane quarter q = warp % 4 holds accumulator rows 32q .. 32q + 31. The records of tile n
    // are formed kFsEpiDelay stages into tile n + 1 (or after the last tile): by then the tile's
    // MMAs have finished, so these warps never hold the stage ring back waiting for them.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    // Forms tile n's records and publishes them; returns true when the four warps stop (a wait
    // ran out here or in another of them). Every warp calls it once per tile, in tile order, so
    // the named barrier sequence stays matched.
    auto epilogue = [&](int n, float ss, bool ok) -> bool {
      const int X = g + n * NG;
      const int b = n & 1;
      if (ok && !__all_sync(0xffffffffu,
                            mbar_wait(&afull[b], static_cast<uint32_t>(n >> 1) & 1u, 47)))
        ok = false;
      if (ok) {
        fs_fence_after();
        uint32_t d[5][16];
        const uint32_t tbase = tmem + static_cast<uint32_t>(b * 128) +
                               (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < 5; ++cc) fs_tmem_ld16(tbase + cc * 16, d[cc]);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        const int64_t t = static_cast<int64_t>(X) * kFsM + row;
        if (t < a.T) {
          float raw[kMix];
#pragma unroll
          for (int c = 0; c < kMix; ++c) {
            const float hi3 = __uint_as_float(d[c / 16][c % 16]);
            const float mid = __uint_as_float(d[(kMix + c) / 16][(kMix + c) % 16]);
            const float lo3 = __uint_as_float(d[(2 * kMix + c) / 16][(2 * kMix + c) % 16]);
            raw[c] = (lo3 + mid) + hi3;
          }
          float4* r4 = reinterpret_cast<float4*>(
              rec_g + ((static_cast<size_t>(n % kFsRing) * kFsM + row) * G + j) * kFsRec);
#pragma unroll
          for (int w = 0; w < 6; ++w)
            r4[w] = make_float4(raw[4 * w], raw[4 * w + 1], raw[4 * w + 2], raw[4 * w + 3]);
          r4[6] = make_float4(ss, 0.f, 0.f, 0.f);
        }
        fs_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aempty[b]);
      }
      // The four warps agree on going on, and their records are published with one
      // release-increment of the tile's counter.
      if (named_bar_or(1, 128, !ok)) return true;
      if (warp == 2 && lane == 0) red_release_add_gpu(a.cnt + X, 1);
      return false;
    };
    int64_t it = 0;
    int pend = -1;  // tile whose records are still to be formed
    float pend_ss = 0.f;
    bool stop = false;
    for (int n = 0; n < ntg && !stop; ++n) {
      bool ok = true;
      float ss0 = 0.f, ss1 = 0.f;
      for (int kb = 0; kb < nb; ++kb, ++it) {
        const int s = static_cast<int>(it % ST);
        const uint32_t ph = static_cast<uint32_t>(it / ST) & 1u;
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, 46))) {
          ok = false;
          break;
        }
        // Row `row` of the swizzled block is its own 128 contiguous bytes (chunks permuted within
        // it); a sum does not depend on the order. Lanes start at different chunks.
        const uint4* rp = reinterpret_cast<const uint4*>(Aring + s * kFsABytes + row * 128);
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
        if (pend >= 0 && kb == kFsEpiDelay) {
          stop = epilogue(pend, pend_ss, true);
          pend = -1;
          if (stop) break;
        }
      }
      if (stop) break;
      if (!ok) {  // the next barrier of the sequence, carrying the failure
        epilogue(pend >= 0 ? pend : n, 0.f, false);
        stop = true;
        break;
      }
      if (pend >= 0) {  // tiles of at most kFsEpiDelay blocks
        stop = epilogue(pend, pend_ss, true);
        if (stop) break;
      }
      pend = n;
      pend_ss = ss0 + ss1;
    }
    if (!stop && pend >= 0) epilogue(pend, pend_ss, true);
  } else if (warp < kFsAggWarp0) {
    // ------------------------------------------------------------------ coefficients
    const int cw = warp - kFsCoefWarp0;
    const int grp = lane / kFsTokLanes;  // token of the pass
    const int gl = lane % kFsTokLanes;   // lane within the token's group
    const int r = lane & 3;  // lanes gl < 4 form the token's quad: pre r, post r, comb row r
    for (int n = cw; n < ntg; n += kFsCoefWarps) {
      const int X = g + n * NG;
      const int slot = n % kFsSlots;
      if (n >= kFsSlots &&
          !__all_sync(0xffffffffu, mbar_wait(&cempty[slot],
                                             static_cast<uint32_t>(n / kFsSlots - 1) & 1u, 48)))
        break;
      if (!__all_sync(0xffffffffu, fs_wait_count(a.cnt + X, G, 49))) break;
      const float* recs = rec_g + static_cast<size_t>(n % kFsRing) * kFsM * G * kFsRec;
      // Owned tokens: l = l0, l0 + G, ... below lim.
      const int l0 = static_cast<int>(((j - (static_cast<int64_t>(n) * kFsM) % G) % G + G) % G);
      const int64_t lim64 = a.T - static_cast<int64_t>(X) * kFsM;
      const int lim = lim64 < kFsM ? static_cast<int>(lim64) : kFsM;
      const int nown = l0 < lim ? (lim - l0 + G - 1) / G : 0;
      for (int p0 = 0; p0 < nown; p0 += kFsTokPerPass) {
        const int k = p0 + grp;
        const bool live = k < nown;
        const int l = l0 + k * G;
        // Lane gl of the token's group adds records gl, gl + kFsTokLanes, ... (all 28 floats of
        // each, in that order); a fixed xor tree then joins the group's lanes. Same order on
        // every run, and every lane of the group ends with the token's sums.
        float acc[kFsRec];
#pragma unroll
        for (int c = 0; c < kFsRec; ++c) acc[c] = 0.f;
        if (live) {
          const float4* rt =
              reinterpret_cast<const float4*>(recs + static_cast<size_t>(l) * G * kFsRec);
          for (int rr = gl; rr < G; rr += 2 * kFsTokLanes) {
            float4 v0[7], v1[7];
            const bool two = rr + kFsTokLanes < G;
#pragma unroll
            for (int c = 0; c < 7; ++c) {
              v0[c] = __ldcg(rt + rr * 7 + c);
              v1[c] = two ? __ldcg(rt + (rr + kFsTokLanes) * 7 + c)
                          : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int c = 0; c < 7; ++c) {
              acc[4 * c] += v0[c].x;
              acc[4 * c + 1] += v0[c].y;
              acc[4 * c + 2] += v0[c].z;
              acc[4 * c + 3] += v0[c].w;
            }
#pragma unroll
            for (int c = 0; c < 7; ++c) {
              acc[4 * c] += v1[c].x;
              acc[4 * c + 1] += v1[c].y;
              acc[4 * c + 2] += v1[c].z;
              acc[4 * c + 3] += v1[c].w;
            }
          }
        }
#pragma unroll
        for (int sh = kFsTokLanes / 2; sh >= 1; sh >>= 1) {
#pragma unroll
          for (int c = 0; c < 25; ++c) acc[c] += __shfl_xor_sync(0xffffffffu, acc[c], sh);
        }
        const int64_t t = static_cast<int64_t>(X) * kFsM + l;
        float cr[4] = {0.f, 0.f, 0.f, 0.f};
        float pre_v = 0.f, post_v = 0.f;
        if (live) {
          const float rstd = __fdiv_rn(
              1.0f, __fsqrt_rn(__fdiv_rn(acc[24], static_cast<float>(a.K)) + a.fp.rms_eps));
          float g0 = acc[0], g1 = acc[4], c0 = acc[8], c1 = acc[9], c2 = acc[10], c3 = acc[11];
          if (r == 1) g0 = acc[1], g1 = acc[5], c0 = acc[12], c1 = acc[13], c2 = acc[14], c3 = acc[15];
          if (r == 2) g0 = acc[2], g1 = acc[6], c0 = acc[16], c1 = acc[17], c2 = acc[18], c3 = acc[19];
          if (r == 3) g0 = acc[3], g1 = acc[7], c0 = acc[20], c1 = acc[21], c2 = acc[22], c3 = acc[23];
          const float lp = fmaf(g0 * rstd, __ldg(a.scale), __ldg(a.base + r));
          const float lq = fmaf(g1 * rstd, __ldg(a.scale + 1), __ldg(a.base + 4 + r));
          const float s2 = __ldg(a.scale + 2);
          cr[0] = fmaf(c0 * rstd, s2, __ldg(a.base + 8 + 4 * r));
          cr[1] = fmaf(c1 * rstd, s2, __ldg(a.base + 9 + 4 * r));
          cr[2] = fmaf(c2 * rstd, s2, __ldg(a.base + 10 + 4 * r));
          cr[3] = fmaf(c3 * rstd, s2, __ldg(a.base + 11 + 4 * r));
          pre_v = sigmoidf_ieee(lp) + a.fp.pre_eps;
          post_v = a.fp.post_mult * sigmoidf_ieee(lq);
        }
        sinkhorn_quad(cr, a.fp.iters, a.fp.sinkhorn_eps);  // every lane takes part
        if (live && gl < 4) {
          a.pre[t * 4 + r] = pre_v;
          a.post[t * 4 + r] = post_v;
#pragma unroll
          for (int c = 0; c < 4; ++c) a.comb[t * 16 + 4 * r + c] = cr[c];
          slot_pre[(slot * kFsMaxOwn + k) * 4 + r] = pre_v;
          if (r == 0) slot_tok[slot * kFsMaxOwn + k] = l;
        }
        __syncwarp();
      }
      if (lane == 0) {
        slot_nown[slot] = nown;
        mbar_arrive(&cfull[slot]);  // release: the hand-over entries above are visible
      }
      __syncwarp();
    }
  } else {
    // ------------------------------------------------------------------ aggregate
    const int at = threadIdx.x - kFsAggWarp0 * 32;
    constexpr int kAggThreads = kFsAggWarps * 32;
    const int64_t H = a.H;
    const int64_t H8 = H / 8;
    for (int n = 0; n < ntg; ++n) {
      const int X = g + n * NG;
      const int slot = n % kFsSlots;
      if (!__all_sync(0xffffffffu,
                      mbar_wait(&cfull[slot], static_cast<uint32_t>(n / kFsSlots) & 1u, 50)))
        break;
      const int nown = slot_nown[slot];
      const int64_t units = static_cast<int64_t>(nown) * H8;
      for (int64_t u0 = at; u0 < units; u0 += 4 * kAggThreads) {
        uint4 rv[4][4];
        uint16_t* yp[4];
        float4 pp[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int64_t u = u0 + e * kAggThreads;
          yp[e] = nullptr;
          if (u < units) {
            const int k = static_cast<int>(u / H8);
            const int64_t v = u - k * H8;
            const int64_t t = static_cast<int64_t>(X) * kFsM + slot_tok[slot * kFsMaxOwn + k];
            pp[e] = *reinterpret_cast<const float4*>(slot_pre + (slot * kFsMaxOwn + k) * 4);
            const uint16_t* rr = a.R + t * 4 * H + v * 8;
#pragma unroll
            for (int i = 0; i < 4; ++i) rv[e][i] = fs_ld_ro(rr + i * H);
            yp[e] = a.y + t * H + v * 8;
          }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          if (yp[e] != nullptr) {
            const uint32_t* r0 = &rv[e][0].x;
            const uint32_t* r1 = &rv[e][1].x;
            const uint32_t* r2 = &rv[e][2].x;
            const uint32_t* r3 = &rv[e][3].x;
            const float4 p4 = pp[e];
            uint32_t o[4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              float lo = p4.x * bf16_lo(r0[c]);
              lo = fmaf(p4.y, bf16_lo(r1[c]), lo);
              lo = fmaf(p4.z, bf16_lo(r2[c]), lo);
              lo = fmaf(p4.w, bf16_lo(r3[c]), lo);
              float hi = p4.x * bf16_hi(r0[c]);
              hi = fmaf(p4.y, bf16_hi(r1[c]), hi);
              hi = fmaf(p4.z, bf16_hi(r2[c]), hi);
              hi = fmaf(p4.w, bf16_hi(r3[c]), hi);
              o[c] = pack_bf16x2(lo, hi);
            }
            st_stream(yp[e], make_uint4(o[0], o[1], o[2], o[3]));
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&cempty[slot]);
    }
  }

  fs_fence_before();
  __syncthreads();
  if (warp == 1) {
    fs_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kFsTmemCols)
                 : "memory");
  }
}

// Zeroes the tile counters; launched right before the fused kernel.
__global__ void pre_fused_zero_kernel(int* cnt, int n) {
  pdl_wait();
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < n; i += gridDim.x * blockDim.x) cnt[i] = 0;
  pdl_trigger();
}

// ------------------------------------------------------------------------------ host side

typedef CUresult (*FsEncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                    const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                    const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                    CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static FsEncodeTiledFn fs_encode_tiled() {
  static FsEncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &p, 12000, cudaEnableDefault,
                                         &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<FsEncodeTiledFn>(p);
    else
      cudaGetLastError();
  });
  return fn;
}

// Returns 0, a negative MHC_ERR_* code, or 1 when this device cannot run the plan's grid with all
// CTAs resident (nothing is launched then).
int launch_pre_fused(const PreArgs& a, cudaStream_t s) {
  const FsPlan plan = fs_plan(a.T, a.H, device_sm_count());
  if (!plan.ok) return 1;
  if (!ensure_smem_limit(reinterpret_cast<const void*>(pre_fused_kernel), plan.smem)) return 1;
  int per_sm = 0;
  if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, pre_fused_kernel, kFsThreads,
                                                    plan.smem) != cudaSuccess ||
      per_sm < 1) {
    cudaGetLastError();
    return 1;
  }
  const int64_t K = 4 * a.H;
  FsEncodeTiledFn fn = fs_encode_tiled();
  if (!fn) return -4;
  CUtensorMap mR;
  {
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K), static_cast<cuuint64_t>(a.T)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K) * 2};
    const cuuint32_t box[2] = {static_cast<cuuint32_t>(kFsKB), static_cast<cuuint32_t>(kFsM)};
    const cuuint32_t estr[2] = {1, 1};
    if (fn(&mR, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(a.R), dims, strides,
           box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
           CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
      return -4;
  }
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  int* cnt = reinterpret_cast<int*>(ws + plan.cnt_off);
  float* rec = reinterpret_cast<float*>(ws + plan.rec_off);

  if (launch_pdl(pre_fused_zero_kernel, dim3(1), dim3(256), 0, s, cnt,
                 static_cast<int>(plan.ntiles)) != cudaSuccess)
    return -4;
  note_launches(1);

  FsArgs fa;
  fa.R = a.R;
  fa.hc_fn = a.hc_fn;
  fa.scale = a.hc_scale;
  fa.base = a.hc_base;
  fa.y = a.y;
  fa.pre = a.pre;
  fa.post = a.post;
  fa.comb = a.comb;
  fa.cnt = cnt;
  fa.rec = rec;
  fa.T = a.T;
  fa.H = a.H;
  fa.K = K;
  fa.KB = static_cast<int>(plan.KB);
  fa.ntiles = static_cast<int>(plan.ntiles);
  fa.G = plan.G;
  fa.NG = plan.NG;
  fa.nbmax = plan.nbmax;
  fa.stages = plan.stages;
  fa.lag = kFsLag;
  fa.fp = FinishParams{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};

  // Cooperative launch: every CTA resident at once (the groups' CTAs wait on one another). Also a
  // programmatic dependent of the zero kernel where the runtime accepts both attributes together.
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(plan.NG * plan.G));
  cfg.blockDim = dim3(kFsThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(plan.smem);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeCooperative;
  attr[0].val.cooperative = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, pre_fused_kernel, mR, fa);
  if (e != cudaSuccess) {
    cudaGetLastError();
    cfg.numAttrs = 1;
    e = cudaLaunchKernelEx(&cfg, pre_fused_kernel, mR, fa);
  }
  if (e != cudaSuccess) {
    cudaGetLastError();
    return -4;
  }
  note_launches(1);
  return 0;
}

}  // namespace mhc
