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
// Kernels (one call, chained with programmatic dependent launch):
//   split   hc_fn [4H][24] fp32 -> Bw [80][4H] bf16 (K contiguous) in the workspace.
//   proj    persistent, one CTA per SM. The work is the (token tile of 256, 64-wide K block)
//           grid flattened tile-major and cut into equal contiguous ranges, one per CTA, so every
//           CTA streams the same number of blocks; a range covers pieces (tile, K interval). Warp 0
//           issues TMA loads of two R sub-tiles [128 x 64] and one Bw tile [80 x 64] (128-byte
//           swizzle) per stage into a 4-stage ring that runs on across pieces; warp 1 issues
//           tcgen05.mma M=128 N=80 K=16 (four per 64-wide K block and sub-tile) into two TMEM
//           accumulators sharing the B tile. A piece is accumulated in sub-pieces of at most 16 K
//           blocks, double-buffered in TMEM (512 columns), so the epilogue of one overlaps the
//           loads of the next; warps 2-5 sum the squares of their token rows from the same
//           shared-memory tiles, add each sub-piece's accumulators (tcgen05.ld) into registers,
//           and after the piece write the record [slot][t][32] = raw[0..23], ss, slot = the
//           piece's rank among its tile's pieces. The CTA holding a tile's last piece writes
//           zero records into the tile's unused slots, so readers sum a fixed number of slots.
//   coef+agg  four tokens per CTA: warp 0 sums each token's slots in order (a lane quad per
//           token), forms rstd, the logits and the pre gates; then the whole CTA writes
//           y = bf16_rn(sum_i pre_i R_i) for those tokens (R read once more, y written once); then
//           warp 0 runs the Sinkhorn and writes post and comb. (Unaligned R / y or H % 8 != 0: the
//           CUDA-core path's finish kernel takes the same records instead.)
#include <cuda.h>

#include <mutex>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kTcM = 128;                          // tokens per MMA (M)
constexpr int kTcSub = 2;                          // MMA sub-tiles per CTA tile sharing one B tile
constexpr int kTcTile = kTcM * kTcSub;             // 256 tokens per CTA tile
constexpr int kTcN = 80;                           // 3 x 24 split columns + 8 zero rows
constexpr int kTcKB = 64;                          // K per block: one 128-byte swizzled row
constexpr int kTcStages = 4;
constexpr int kTcABytes = kTcM * kTcKB * 2;        // 16384 per sub-tile
constexpr int kTcBBytes = kTcN * kTcKB * 2;        // 10240
constexpr int kTcStageBytes = kTcSub * kTcABytes + kTcBBytes;  // 43008 = 42 x 1024
constexpr int kTcThreads = 192;
constexpr int kTcTmemCols = 512;                   // 2 buffers x 2 sub-tiles x 128 columns
constexpr int kTcSmem = 1024 + kTcStages * kTcStageBytes + 256;
// The backward's projection also carries d_y: it walks a tile's K blocks column-block-major (the
// four streams of a 64-column block consecutively) and keeps the block's d_y tile [256 x 64] in
// one of two slots for those four stages; three stages.
constexpr int kTcDyStages = 3;
constexpr int kTcDyBytes = kTcSub * kTcABytes;  // 32 KB
constexpr int kTcDySmem = 1024 + kTcDyStages * kTcStageBytes + 2 * kTcDyBytes + 256;
static_assert(kTcDySmem <= 227 * 1024, "shared memory");
constexpr int64_t kTcMaxCtas = 148;                // most CTAs the projection plan uses
constexpr int64_t kTcMinBlocks = 8;                // K blocks per CTA at least (pipeline fill)
// The tensor-core accumulator is restarted every kTcSubBlocks K blocks of a piece and the sub-piece
// sums are added in registers: shorter accumulation chains in TMEM keep the projection's fp32
// rounding error well inside the coefficient tolerance over K = 4H = 28672.
constexpr int kTcSubBlocks = 16;
constexpr int kTcAccDelay = 2;  // stages into the next sub-piece before a finished one is added

// Work plan of the projection: W = ntiles * kblocks block-tiles over P CTAs; CTA c takes
// [c W / P, (c + 1) W / P). A tile's K range is cut into at most S pieces.
struct TcPlan {
  int64_t ntiles, kblocks, W, P, S;
  size_t bw_bytes;  // workspace bytes of Bw, rounded to 1 KB
};

// `sms` is the device's SM count at launch; workspace sizing uses the largest plan (kTcMaxCtas),
// which never needs fewer slots than a plan over fewer CTAs.
static TcPlan tc_plan(int64_t T, int64_t H, int64_t sms = kTcMaxCtas) {
  TcPlan p;
  const int64_t K = 4 * H;
  p.ntiles = (T + kTcTile - 1) / kTcTile;
  p.kblocks = (K + kTcKB - 1) / kTcKB;
  p.W = p.ntiles * p.kblocks;
  p.P = p.W / kTcMinBlocks;
  if (p.P > kTcMaxCtas) p.P = kTcMaxCtas;
  if (p.P > sms) p.P = sms;
  if (p.P < 1) p.P = 1;
  // A tile spans kblocks consecutive units; a CTA range holds at least floor(W / P) of them, so a
  // tile meets at most floor(kblocks P / W) + 2 ranges.
  p.S = p.kblocks * p.P / p.W + 2;
  if (p.S > p.P) p.S = p.P;
  p.bw_bytes = (static_cast<size_t>(kTcN) * K * 2 + 1023) / 1024 * 1024;
  return p;
}

// First CTA whose range contains flattened unit x.
__host__ __device__ __forceinline__ int64_t tc_first_cta(int64_t x, int64_t P, int64_t W) {
  return ((x + 1) * P - 1) / W;
}

bool pre_tc_supported(int64_t T, int64_t H) {
  // TMA needs 16-byte global strides: rows of R (8H bytes) and of Bw (8H bytes).
  return T >= 1 && H >= 2 && H % 2 == 0 && (T + kTcTile - 1) / kTcTile <= 0x7fffffff &&
         (4 * H + kTcKB - 1) / kTcKB <= 0x7fffffff;
}

size_t pre_tc_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0 || H % 2 != 0) return 0;
  const TcPlan p = tc_plan(T, H);
  return p.bw_bytes + static_cast<size_t>(p.S) * static_cast<size_t>(T) * 32 * sizeof(float);
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
__device__ __forceinline__ void split_hc_fn_row(const float* __restrict__ W,
                                                uint16_t* __restrict__ Bw, int64_t K, int64_t k) {
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

__global__ void __launch_bounds__(256) pre_tc_split_kernel(const float* __restrict__ W,
                                                           uint16_t* __restrict__ Bw, int64_t K) {
  pdl_wait();  // the previous call's projection may still read Bw
  pdl_trigger();
  for (int64_t k = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; k < K;
       k += (int64_t)gridDim.x * blockDim.x)
    split_hc_fn_row(W, Bw, K, k);
}

// kDy (the pre-map backward's recomputation): the stages also hold the d_y columns of each K
// block, and the sum-of-squares warps form d_pre's term sum_h d_y R_i of each token row per stream
// i, into record floats 28..31 (requires H % 64 == 0, so that a K block lies in one stream).
template <bool kDy>
__global__ void __launch_bounds__(kTcThreads, 1) pre_tc_proj_kernel(
    const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmB,
    const __grid_constant__ CUtensorMap tmDy, float* __restrict__ part, int64_t T, int64_t W,
    int KB, int S, int64_t H) {
  constexpr int ST = kDy ? kTcDyStages : kTcStages;
  constexpr int SB = kTcStageBytes;
  constexpr int kDyArea = kDy ? 2 * kTcDyBytes : 0;  // d_y slots after the stages
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* dyslots = smem + ST * SB;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + ST * SB + kDyArea);
  uint64_t* empty = full + ST;
  uint64_t* afull = empty + ST;  // [2] accumulator buffer b complete (MMA commit)
  uint64_t* aempty = afull + 2;         // [2] accumulator buffer b read out (4 warps)
  uint64_t* done = aempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);
  static_assert((2 * ST + 5) * 8 + 4 <= 256, "barrier area");

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t lo = c * W / P, hi = (c + 1) * W / P;
  // kDy: the kb-th block of a tile is stream kb % 4 of column block kb / 4 (KB = 4 H / 64);
  // otherwise blocks follow k = i H + h.
  const int hbk = KB / 4;
  auto pkb = [&](int kb) -> int { return kDy ? (kb & 3) * hbk + (kb >> 2) : kb; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < ST; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1 + 4);  // MMA commit + one arrival per sum-of-squares warp
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], 4);
    }
    mbar_init(done, 1);
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
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    if (lane == 0) {
      int64_t n = 0, ng = -1;  // ng: d_y groups loaded (kDy)
      bool ok = true;
      for (int64_t u = lo; u < hi && ok;) {
        const int64_t tile = u / KB;
        const int kbs = static_cast<int>(u - tile * KB);
        const int kbe = static_cast<int>(min(static_cast<int64_t>(KB), kbs + (hi - u)));
        for (int kb = kbs; kb < kbe; ++kb, ++n) {
          const int s = static_cast<int>(n % ST);
          const uint32_t ph = static_cast<uint32_t>(n / ST) & 1u;
          if (n >= ST && !mbar_wait(&empty[s], ph ^ 1u, 10)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + s * SB;
          // kDy: a block that opens a column block (or a piece) also brings that column block's
          // d_y tile, into the slot the group after next will reuse (by then the sum-of-squares
          // warps are past this group: the ring is shorter than a group).
          const bool newg = kDy && ((kb & 3) == 0 || kb == kbs);
          if (newg) ++ng;
          mbar_arrive_expect_tx(&full[s], SB + (newg ? kTcDyBytes : 0));
          const int x = pkb(kb) * kTcKB;
#pragma unroll
          for (int v = 0; v < kTcSub; ++v)
            tma_load_2d(st + v * kTcABytes, &tmR, x,
                        static_cast<int>(tile * kTcTile + v * kTcM), &full[s]);
          tma_load_2d(st + kTcSub * kTcABytes, &tmB, x, 0, &full[s]);
          if (newg) {
            uint8_t* ds = dyslots + (ng & 1) * kTcDyBytes;
#pragma unroll
            for (int v = 0; v < kTcSub; ++v)
              tma_load_2d(ds + v * kTcABytes, &tmDy, (kb >> 2) * kTcKB,
                          static_cast<int>(tile * kTcTile + v * kTcM), &full[s]);
          }
        }
        u += kbe - kbs;
      }
      if (!ok) {  // do not leave while copies into shared memory are in flight
        for (int64_t i = n - ST; i < n; ++i)
          if (i >= 0)
            mbar_wait(&full[i % ST], static_cast<uint32_t>(i / ST) & 1u, 15);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t n = 0;
      int64_t sp = 0;  // sub-pieces issued (accumulator buffer sp & 1)
      bool ok = true;
      uint32_t dt = tmem;
      for (int64_t u = lo; u < hi && ok;) {
        const int64_t tile = u / KB;
        const int kbs = static_cast<int>(u - tile * KB);
        const int kbe = static_cast<int>(min(static_cast<int64_t>(KB), kbs + (hi - u)));
        for (int kb = kbs; kb < kbe; ++kb, ++n) {
          const int ks = (kb - kbs) % kTcSubBlocks;  // position within the sub-piece
          if (ks == 0) {
            const int b = static_cast<int>(sp & 1);
            if (sp >= 2 && !mbar_wait(&aempty[b], static_cast<uint32_t>((sp >> 1) - 1) & 1u, 16)) {
              ok = false;
              break;
            }
            tc_fence_after();
            dt = tmem + static_cast<uint32_t>(b * kTcSub * kTcM);
          }
          const int s = static_cast<int>(n % ST);
          const uint32_t ph = static_cast<uint32_t>(n / ST) & 1u;
          if (!mbar_wait(&full[s], ph, 11)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a = smem_u32(smem + s * SB);
          const uint64_t bdesc = sw128_desc(a + kTcSub * kTcABytes);
#pragma unroll
          for (int v = 0; v < kTcSub; ++v) {
            const uint64_t adesc = sw128_desc(a + v * kTcABytes);
#pragma unroll
            for (int k = 0; k < kTcKB / 16; ++k)  // +32 bytes along the swizzled row per K=16 step
              umma_bf16(dt + static_cast<uint32_t>(v * kTcM), adesc + 2 * k, bdesc + 2 * k,
                        (ks > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&empty[s]);
          if (kb + 1 == kbe || ks + 1 == kTcSubBlocks) {
            umma_commit(&afull[sp & 1]);
            ++sp;
          }
        }
        u += kbe - kbs;
      }
      // Every issued MMA has finished before TMEM is released.
      umma_commit(done);
      mbar_wait(done, 0, 14);
    }
  } else {
    // Warps 2..5: TMEM lane quarter q = warp % 4 holds rows 32q..32q+31 of each sub-tile's
    // accumulator; the same thread sums the squares of those rows (one per sub-tile).
    const int q_lane = warp & 3;
    const int row = q_lane * 32 + lane;
    int64_t n = 0, ng = -1;  // ng: d_y groups seen (kDy), as the producer counts them
    int64_t sp = 0;     // sub-pieces the MMA warp has been asked to finish
    int64_t pend = -1;  // finished sub-piece whose accumulators are not yet added
    bool ok = true;
    float racc[kTcSub][kMix];
    // Adds sub-piece q's accumulators (TMEM buffer q & 1) to the piece's sums; false on timeout.
    auto add_sub = [&](int64_t q) -> bool {
      const int b = static_cast<int>(q & 1);
      if (!__all_sync(0xffffffffu, mbar_wait(&afull[b], static_cast<uint32_t>(q >> 1) & 1u, 13)))
        return false;
      tc_fence_after();
#pragma unroll
      for (int v = 0; v < kTcSub; ++v) {
        uint32_t d[5][16];
        const uint32_t tbase = tmem + static_cast<uint32_t>((b * kTcSub + v) * kTcM) +
                               (static_cast<uint32_t>(q_lane * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < 5; ++cc) tmem_ld16(tbase + cc * 16, d[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kMix; ++j) {
          const float hi3 = __uint_as_float(d[j / 16][j % 16]);
          const float mid = __uint_as_float(d[(kMix + j) / 16][(kMix + j) % 16]);
          const float lo3 = __uint_as_float(d[(2 * kMix + j) / 16][(2 * kMix + j) % 16]);
          racc[v][j] += (lo3 + mid) + hi3;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&aempty[b]);
      return true;
    };
    for (int64_t u = lo; u < hi && ok;) {
      const int64_t tile = u / KB;
      const int kbs = static_cast<int>(u - tile * KB);
      const int kbe = static_cast<int>(min(static_cast<int64_t>(KB), kbs + (hi - u)));
      float ss0[kTcSub], ss1[kTcSub];
      float dpv[kTcSub][4];  // kDy: sum_h d_y R_i of the row, per stream i
#pragma unroll
      for (int v = 0; v < kTcSub; ++v) {
        ss0[v] = ss1[v] = 0.f;
#pragma unroll
        for (int j = 0; j < kMix; ++j) racc[v][j] = 0.f;
#pragma unroll
        for (int i = 0; i < 4; ++i) dpv[v][i] = 0.f;
      }
      for (int kb = kbs; kb < kbe; ++kb, ++n) {
        const int s = static_cast<int>(n % ST);
        const uint32_t ph = static_cast<uint32_t>(n / ST) & 1u;
        // Every lane waits; the warp continues only if all of them saw the stage (warp-uniform,
        // so the __syncwarp and the .sync.aligned TMEM loads below are never reached divergently).
        if (!__all_sync(0xffffffffu, mbar_wait(&full[s], ph, 12))) {
          ok = false;
          break;
        }
        if (kDy && ((kb & 3) == 0 || kb == kbs)) ++ng;  // this block's d_y slot: ng & 1
#pragma unroll
        for (int v = 0; v < kTcSub; ++v) {
          // Row `row` of the swizzled tile is its own 128 contiguous bytes (chunks permuted within
          // it), and a sum does not depend on element order. Each lane starts at a different
          // 16-byte chunk, so the 8 lanes of a load phase hit 8 different bank groups. The d_y
          // tile has the same geometry and swizzle, so chunk c of both rows holds the same columns.
          const uint4* rp = reinterpret_cast<const uint4*>(smem + s * SB +
                                                           v * kTcABytes + row * 128);
          float dsum = 0.f;
#pragma unroll
          for (int cc = 0; cc < 8; ++cc) {
            const uint4 w = rp[cc ^ (lane & 7)];
            const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
            uint32_t g4[4] = {0u, 0u, 0u, 0u};
            if constexpr (kDy) {
              const uint4 g = reinterpret_cast<const uint4*>(
                  dyslots + (ng & 1) * kTcDyBytes + v * kTcABytes + row * 128)[cc ^ (lane & 7)];
              g4[0] = g.x, g4[1] = g.y, g4[2] = g.z, g4[3] = g.w;
            }
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float x0 = bf16_lo(w4[e]), x1 = bf16_hi(w4[e]);
              ss0[v] = fmaf(x0, x0, ss0[v]);
              ss1[v] = fmaf(x1, x1, ss1[v]);
              if constexpr (kDy) {
                dsum = fmaf(bf16_lo(g4[e]), x0, dsum);
                dsum = fmaf(bf16_hi(g4[e]), x1, dsum);
              }
            }
          }
          if constexpr (kDy) {
            const int si = kb & 3;  // the block's stream
#pragma unroll
            for (int i = 0; i < 4; ++i)
              if (si == i) dpv[v][i] += dsum;
          }
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(&empty[s]);
        const int ks = (kb - kbs) % kTcSubBlocks;
        // A finished sub-piece is added a few stages into the next one (its MMAs are done by
        // then, so this never holds the stage ring back); the last one at the end of the piece.
        if (pend >= 0 && ks == kTcAccDelay) {
          if (!add_sub(pend)) {
            ok = false;
            break;
          }
          pend = -1;
        }
        if (kb + 1 == kbe || ks + 1 == kTcSubBlocks) {
          if (pend >= 0 && !add_sub(pend)) {
            ok = false;
            break;
          }
          pend = sp++;
        }
      }
      if (ok && pend >= 0 && !add_sub(pend)) ok = false;
      pend = -1;
      if (!ok) break;
      const int64_t slot = c - tc_first_cta(tile * KB, P, W);
      const bool last_piece = (kbe == KB);
#pragma unroll
      for (int v = 0; v < kTcSub; ++v) {
        const int64_t t = tile * kTcTile + v * kTcM + row;
        if (t < T) {
          float4* rec = reinterpret_cast<float4*>(part + (slot * T + t) * 32);
#pragma unroll
          for (int w = 0; w < 6; ++w)
            rec[w] = make_float4(racc[v][4 * w], racc[v][4 * w + 1], racc[v][4 * w + 2],
                                 racc[v][4 * w + 3]);
          rec[6] = make_float4(ss0[v] + ss1[v], 0.f, 0.f, 0.f);
          if constexpr (kDy) rec[7] = make_float4(dpv[v][0], dpv[v][1], dpv[v][2], dpv[v][3]);
          if (last_piece) {
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int64_t sl = slot + 1; sl < S; ++sl) {
              float4* zr = reinterpret_cast<float4*>(part + (sl * T + t) * 32);
#pragma unroll
              for (int w = 0; w < (kDy ? 8 : 7); ++w) zr[w] = z;
            }
          }
        }
      }
      u += kbe - kbs;
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

// y = bf16_rn(sum_i pre_i * R_i): one thread per (token, 8 columns), a streaming pass (R read once,
// y written once). Requires H % 8 == 0 and 16-byte aligned R, y and pre.
__global__ void __launch_bounds__(256) pre_agg_vec8_kernel(const uint16_t* __restrict__ R,
                                                           const float* __restrict__ pre,
                                                           uint16_t* __restrict__ y, int64_t T,
                                                           int64_t H8) {
  const int64_t total = T * H8;
  const int64_t H = H8 * 8;
  pdl_wait();
  pdl_trigger();
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
      float a = p4.x * bf16_lo(r0[e]);
      a = fmaf(p4.y, bf16_lo(r1[e]), a);
      a = fmaf(p4.z, bf16_lo(r2[e]), a);
      a = fmaf(p4.w, bf16_lo(r3[e]), a);
      float b = p4.x * bf16_hi(r0[e]);
      b = fmaf(p4.y, bf16_hi(r1[e]), b);
      b = fmaf(p4.z, bf16_hi(r2[e]), b);
      b = fmaf(p4.w, bf16_hi(r3[e]), b);
      o[e] = pack_bf16x2(a, b);
    }
    st_plain(y + t * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));
  }
}

// Coefficients and aggregate in one kernel, kCaTok tokens per CTA (the split chain's last step).
// Warp 0 forms the tokens' logits from the slot records (one lane quad per token) and their pre
// gates; after a block barrier all 256 threads write y for those tokens with 16-byte accesses (eight
// CTAs per SM keep the loads in flight); then warp 0 runs the tokens' Sinkhorn and writes post and comb, while
// the SM's other CTAs keep the stream going. One kernel fewer in the chain than coef + aggregate.
// Requires H % 8 == 0 and 16-byte aligned R and y.
constexpr int kCaTok = 4;  // measured: 4 beats 2, 8 and 16 at T = 3072 and 8192
static_assert(kCaTok <= 8, "warp 0 holds one lane quad per token");

__global__ void __launch_bounds__(256, 8) pre_tc_coef_agg_kernel(
    const uint16_t* __restrict__ R, const float* __restrict__ part, int nslot,
    const float* __restrict__ scale, const float* __restrict__ base, uint16_t* __restrict__ y,
    float* __restrict__ pre, float* __restrict__ post, float* __restrict__ comb, int64_t T,
    int64_t H8, int64_t K, FinishParams fp) {
  __shared__ float4 spre[kCaTok];
  __shared__ float slog[32][5];  // comb row logits and post logit of each lane of warp 0
  pdl_wait();
  pdl_trigger();
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * kCaTok;
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int r = lane & 3;
    const int qd = lane >> 2;  // token of this quad within the CTA (quads kCaTok.. are idle)
    const int64_t t = t0 + qd;
    const bool live = qd < kCaTok && t < T;
    const int64_t tt = live ? t : 0;
    float4 g0 = make_float4(0.f, 0.f, 0.f, 0.f), g1 = g0, gc = g0;
    float g6 = 0.f;
    for (int s = 0; s < nslot; ++s) {
      const float4* rec = reinterpret_cast<const float4*>(part + (s * T + tt) * 32);
      const float4 a0 = __ldg(rec), a1 = __ldg(rec + 1), ac = __ldg(rec + 2 + r);
      const float a6 = __ldg(reinterpret_cast<const float*>(rec + 6));
      g0.x += a0.x, g0.y += a0.y, g0.z += a0.z, g0.w += a0.w;
      g1.x += a1.x, g1.y += a1.y, g1.z += a1.z, g1.w += a1.w;
      gc.x += ac.x, gc.y += ac.y, gc.z += ac.z, gc.w += ac.w;
      g6 += a6;
    }
    const float rstd =
        __fdiv_rn(1.0f, __fsqrt_rn(__fdiv_rn(g6, static_cast<float>(K)) + fp.rms_eps));
    const float g0r = r == 0 ? g0.x : r == 1 ? g0.y : r == 2 ? g0.z : g0.w;
    const float g1r = r == 0 ? g1.x : r == 1 ? g1.y : r == 2 ? g1.z : g1.w;
    const float lp = fmaf(g0r * rstd, __ldg(scale), __ldg(base + r));
    slog[lane][4] = fmaf(g1r * rstd, __ldg(scale + 1), __ldg(base + 4 + r));
    const float s2 = __ldg(scale + 2);
    slog[lane][0] = fmaf(gc.x * rstd, s2, __ldg(base + 8 + 4 * r));
    slog[lane][1] = fmaf(gc.y * rstd, s2, __ldg(base + 9 + 4 * r));
    slog[lane][2] = fmaf(gc.z * rstd, s2, __ldg(base + 10 + 4 * r));
    slog[lane][3] = fmaf(gc.w * rstd, s2, __ldg(base + 11 + 4 * r));
    const float pv = sigmoidf_ieee(lp) + fp.pre_eps;
    if (live) pre[t * 4 + r] = pv;
    if (qd < kCaTok) reinterpret_cast<float*>(spre)[qd * 4 + r] = pv;
  }
  __syncthreads();
  const int64_t ntok = min(static_cast<int64_t>(kCaTok), T - t0);
  const int64_t units = ntok * H8;
  const int64_t H = H8 * 8;
  for (int64_t u = threadIdx.x; u < units; u += 256) {
    const int64_t k = u / H8;
    const int64_t v = u - k * H8;
    const uint16_t* rr = R + (t0 + k) * 4 * H + v * 8;
    uint4 rv[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) rv[i] = ld_stream_ro(rr + i * H);
    const float4 p4 = spre[k];
    const uint32_t* r0 = &rv[0].x;
    const uint32_t* r1 = &rv[1].x;
    const uint32_t* r2 = &rv[2].x;
    const uint32_t* r3 = &rv[3].x;
    uint32_t o[4];
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      float a = p4.x * bf16_lo(r0[c]);
      a = fmaf(p4.y, bf16_lo(r1[c]), a);
      a = fmaf(p4.z, bf16_lo(r2[c]), a);
      a = fmaf(p4.w, bf16_lo(r3[c]), a);
      float b = p4.x * bf16_hi(r0[c]);
      b = fmaf(p4.y, bf16_hi(r1[c]), b);
      b = fmaf(p4.z, bf16_hi(r2[c]), b);
      b = fmaf(p4.w, bf16_hi(r3[c]), b);
      o[c] = pack_bf16x2(a, b);
    }
    st_stream(y + (t0 + k) * H + v * 8, make_uint4(o[0], o[1], o[2], o[3]));  // not re-read here
  }
  if (threadIdx.x < 32) {  // warp 0 wrote slog before the barrier above
    const int lane = threadIdx.x;
    const int r = lane & 3;
    const int qd = lane >> 2;
    const int64_t t = t0 + qd;
    const bool live = qd < kCaTok && t < T;
    float cr[4] = {0.f, 0.f, 0.f, 0.f};
    if (qd < kCaTok) {
#pragma unroll
      for (int c = 0; c < 4; ++c) cr[c] = slog[lane][c];
    }
    sinkhorn_quad(cr, fp.iters, fp.sinkhorn_eps);  // every lane of warp 0 takes part
    if (live) {
      post[t * 4 + r] = fp.post_mult * sigmoidf_ieee(slog[lane][4]);
#pragma unroll
      for (int c = 0; c < 4; ++c) comb[t * 16 + 4 * r + c] = cr[c];
    }
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

// Split + projection: records [S][T][32] (raw[24], ss) in the workspace after Bw. Returns 0 or a
// negative MHC_ERR_* code; *part_out / *nrec_out receive the records and their slot count.
int launch_tc_projection(const PreArgs& a, cudaStream_t s, float** part_out, int* nrec_out,
                         const uint16_t* dy) {
  const TcPlan plan = tc_plan(a.T, a.H, device_sm_count());
  const int64_t K = 4 * a.H;
  uint8_t* ws = static_cast<uint8_t*>(a.workspace);
  uint16_t* Bw = reinterpret_cast<uint16_t*>(ws);
  float* part = reinterpret_cast<float*>(ws + plan.bw_bytes);

  CUtensorMap mR, mB, mDy;
  if (!make_map(&mR, a.R, K, a.T, kTcM) || !make_map(&mB, Bw, K, kTcN, kTcN)) return -4;
  if (dy != nullptr && !make_map(&mDy, dy, a.H, a.T, kTcM)) return -4;
  if (dy == nullptr) mDy = mR;  // unused by the form without d_y

  if (!ensure_smem_limit(reinterpret_cast<const void*>(pre_tc_proj_kernel<false>), kTcSmem) ||
      !ensure_smem_limit(reinterpret_cast<const void*>(pre_tc_proj_kernel<true>), kTcDySmem))
    return -4;

  const int64_t sb = (K + 255) / 256;
  const int split_blocks = static_cast<int>(sb < 4096 ? sb : 4096);
  if (launch_pdl(pre_tc_split_kernel, dim3(split_blocks), dim3(256), 0, s,
                 static_cast<const float*>(a.hc_fn), Bw, K) != cudaSuccess)
    return -4;
  note_launches(1);

  const cudaError_t e =
      dy != nullptr
          ? launch_pdl(pre_tc_proj_kernel<true>, dim3(static_cast<unsigned>(plan.P)),
                       dim3(kTcThreads), static_cast<size_t>(kTcDySmem), s, mR, mB, mDy, part,
                       a.T, plan.W, static_cast<int>(plan.kblocks), static_cast<int>(plan.S), a.H)
          : launch_pdl(pre_tc_proj_kernel<false>, dim3(static_cast<unsigned>(plan.P)),
                       dim3(kTcThreads), static_cast<size_t>(kTcSmem), s, mR, mB, mDy, part,
                       a.T, plan.W, static_cast<int>(plan.kblocks), static_cast<int>(plan.S), a.H);
  if (e != cudaSuccess) return -4;
  note_launches(1);
  *part_out = part;
  *nrec_out = static_cast<int>(plan.S);
  return 0;
}

int launch_pre_tc(const PreArgs& a, cudaStream_t s) {
  float* part = nullptr;
  int nrec = 0;
  const int r = launch_tc_projection(a, s, &part, &nrec);
  if (r != 0) return r;

  const FinishParams fp{a.iters, a.sinkhorn_eps, a.rms_eps, a.pre_eps, a.post_mult};
  const bool vec = aligned16(a.R) && aligned16(a.y) && (a.H % 8 == 0);
  if (vec) {
    const int64_t cb = (a.T + kCaTok - 1) / kCaTok;
    if (cb > 0x7fffffff) return -5;
    if (launch_pdl(pre_tc_coef_agg_kernel, dim3(static_cast<unsigned>(cb)), dim3(256), 0, s, a.R,
                   static_cast<const float*>(part), nrec, a.hc_scale, a.hc_base, a.y, a.pre,
                   a.post, a.comb, a.T, a.H / 8, 4 * a.H, fp) != cudaSuccess)
      return -4;
  } else {
    const int64_t nhb = (a.H + kAggCols - 1) / kAggCols;
    if (a.T > 0x7fffffff || 1 + nhb > 65535) return -5;
    const dim3 g2(static_cast<unsigned>(a.T), static_cast<unsigned>(1 + nhb));
    if (launch_pdl(pre_cc_finish_kernel<false>, g2, dim3(256), 0, s, a.R, part,
                   static_cast<int64_t>(nrec),
                   a.hc_scale, a.hc_base, a.y, a.pre, a.post, a.comb, a.T, a.H, fp) != cudaSuccess)
      return -4;
  }
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? 0 : -4;
}

}  // namespace mhc
