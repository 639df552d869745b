// Pre-map backward, d_R and d_hc_fn on tcgen05 tensor cores, in one pass over R.
//
// d_R[t][k] = sum_j d_raw[t][j] hc_fn[k][j] + 2 R[t][k] d_ss[t] + pre_i[t] d_y[t][h], k = i*H + h
// d_hc_fn[k][j] = sum_t R[t][k] d_raw[t][j]
// (the chain rule through raw = R_flat . hc_fn, the sum of squares and y = sum_i pre_i R_i;
// "FlashInfer mHC module deep dive" §3.4 / §5.2 forward). Both contractions have 24 as one
// dimension: on CUDA cores they are bound by issue; on tensor cores the kernel is bound by its
// traffic (R and d_y read once, d_R written).
//
// Operands (written by pre_bwd_split_kernel, bf16, 128 columns per row, zero past 72; the d_R
// MMAs read columns 0..79: four K=16 steps in a 128-byte-swizzled box, one in a 32-byte-swizzled
// box):
//   A[t] = [hi(d_raw) | lo(d_raw) | hi(d_raw)],  B[k] = [hi(w) | hi(w) | lo(w)],  w = hc_fn[k][.]
// so A.B = hi.hi + lo.hi + hi.lo of each product, exact in the fp32 accumulator; the dropped
// lo.lo term and the split's remainders are below 2^-15 of each product. The first 48 columns of
// A, [hi | lo] of d_raw, are also d_hc_fn's B operand (read MN-major: tokens along K), with R's
// staged tile as its A operand (MN-major: 128 columns k along M), so each d_hc_fn product is
// R.hi + R.lo, exact in fp32 (R is exact in bf16; hi + lo leaves below 2^-16 of d_raw).
//
// pre_bwd_drw_kernel: persistent, one CTA per SM. Work items (column block hc of 128 columns
// within a stream, token tile tt of 128, stream i), numbered with i fastest, so the four items of
// an (hc, tt) group share one d_y tile and one A tile; the list is cut into equal contiguous
// ranges, one per CTA. A unit is (hc, chunk of kDrwChunk token tiles); a CTA's items inside one
// unit form a piece, whose rank among the unit's CTAs is its partial slot.
//   warp 0      TMA: the group's d_y tile (two buffers), and per item the R tile and the B tile
//               (rings of three and two: an R slot is free once its d_R has been stored, a B slot
//               once its MMAs have read it); all [128 x 64] boxes with the 128-byte swizzle.
//   warp 1      tcgen05.mma: per item, eight M=128 N=64 K=16 steps of d_hc_fn into stream i's
//               accumulator (restarted at the piece's first item of that stream), then five
//               M=128 N=128 K=16 steps of d_R into one of two accumulators (TMEM: 2 x 128 + 4 x
//               64 columns). It also loads the A tile, once the MMAs on the previous one are done.
//   warps 2-5   epilogue, thread = token row (its TMEM lane): 64 accumulator columns at a time
//               (tcgen05.ld), R and d_y from the staged tiles, out = bf16_rn(fma(pre_i, d_y,
//               fma(2 d_ss, R, acc))) written over R in place (after the item's MMAs, which read
//               R, have completed). At a piece's end, thread = column k: the partial
//               [ck * S + slot][k][24] = lo + hi columns of each stream's accumulator (zero for a
//               stream the piece did not reach); the CTA holding a unit's last item zero-fills its
//               unused slots. pre_bwd_dw_sum_kernel adds the slices in order.
//   warp 6      stores each finished d_R tile with a TMA bulk-tensor store and releases its R slot
//               once the store has read it (the epilogue warps go on to the next item meanwhile).
// Every wait is bounded; copies in flight are drained and stores completed before exit.
// Requires H % 128 == 0, 16-byte aligned R, d_y (when given; absent, its term is zero and no d_y
// tile is loaded), d_R and workspace.
// The TMA, descriptor, MMA and TMEM helpers and the tensor-map encoder are mhc_pre_tc.cu's (same
// translation unit).
#include <cuda.h>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kDrM = 128;                      // tokens per tile
constexpr int kDrN = 128;                      // columns of d_R per item
constexpr int kDrKd = 128;                     // split inner dimension (72 used), two swizzle atoms
constexpr int kDrAtom = 128 * 64 * 2;          // one [128 x 64] bf16 box: 16 KB
constexpr int kDrTile = 2 * kDrAtom;           // [128 x 128] bf16: 32 KB
// A and B operand tiles: split columns 0..63 as one [128 x 64] box with the 128-byte swizzle and
// columns 64..79 as a [128 x 16] box with the 32-byte swizzle (columns 80..127 are never loaded).
constexpr int kDrAtomNarrow = 128 * 16 * 2;    // 4 KB
constexpr int kDrOpTile = kDrAtom + kDrAtomNarrow;  // 20 KB
constexpr int kDrRSlots = 3;                   // R ring (the HBM stream); d_R is staged in place
constexpr int kDrBSlots = 2;                   // B ring (L2; freed as soon as the MMAs read it)
constexpr int kDrOffA = 0;
constexpr int kDrOffDy = kDrOffA + kDrOpTile;          // two buffers
constexpr int kDrOffB = kDrOffDy + 2 * kDrTile;
constexpr int kDrOffR = kDrOffB + kDrBSlots * kDrOpTile;
constexpr int kDrOffBars = kDrOffR + kDrRSlots * kDrTile;  // 225280
constexpr int kDrSmem = 1024 + kDrOffBars + 256;
constexpr int kDrThreads = 224;
constexpr int kDrTmemCols = 512;
// d_hc_fn: accumulators of the four streams at columns 256 + 64 i (N = 64: split columns
// [hi | lo | hi(0..15)] of d_raw; the last 16 are not read), restarted every kDrwChunk token tiles.
constexpr int kDrwN = 64;
constexpr int kDrwCol0 = 2 * 128;
constexpr int kDrwChunk = 64;
// kind::f16, D fp32, A and B bf16, both MN-major (bits 15, 16), N = 64, M = 128.
constexpr uint32_t kDrwIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) | (1u << 16) |
                               (static_cast<uint32_t>(kDrwN >> 3) << 17) |
                               (static_cast<uint32_t>(128 >> 4) << 24);
constexpr uint32_t kDrIdesc = (1u << 4) | (1u << 7) | (1u << 10) |
                              (static_cast<uint32_t>(kDrN >> 3) << 17) |
                              (static_cast<uint32_t>(kDrM >> 4) << 24);
static_assert(kDrSmem <= 227 * 1024, "shared memory");

bool pre_bwd_dr_tc_supported(int64_t T, int64_t H) {
  return T >= 1 && H >= 128 && H % 128 == 0 && (T + kDrM - 1) / kDrM <= (int64_t(1) << 24);
}

// Work plan: W items over P CTAs; S = most CTAs one unit meets (a unit holds at most
// min(ntt, kDrwChunk) * 4 consecutive items and a range at least floor(W / P)).
struct DrPlan {
  int64_t ntt, nhc, W, nck, P, S;
};

static DrPlan dr_plan(int64_t T, int64_t H, int64_t sms) {
  DrPlan p;
  p.ntt = (T + kDrM - 1) / kDrM;
  p.nhc = H / kDrN;
  p.W = p.ntt * p.nhc * 4;
  p.nck = (p.ntt + kDrwChunk - 1) / kDrwChunk;
  p.P = sms < 148 ? sms : 148;
  if (p.P > p.W) p.P = p.W;
  if (p.P < 1) p.P = 1;
  const int64_t per_unit = (p.ntt < kDrwChunk ? p.ntt : kDrwChunk) * 4;
  p.S = per_unit * p.P / p.W + 2;
  if (p.S > p.P) p.S = p.P;
  return p;
}

// A and B operands, then the d_hc_fn partials (a plan over fewer SMs never needs more slots).
size_t pre_bwd_dr_tc_workspace_bytes(int64_t T, int64_t H) {
  if (!pre_bwd_dr_tc_supported(T, H)) return 0;
  auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
  const DrPlan p = dr_plan(T, H, 148);
  return up(static_cast<size_t>(T) * kDrKd * 2) + up(static_cast<size_t>(4 * H) * kDrKd * 2) +
         up(static_cast<size_t>(p.nck * p.S) * static_cast<size_t>(4 * H) * kMix * 4);
}

__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}

__device__ __forceinline__ void dr_umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kDrIdesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor: K-major, 32-byte swizzle, 8-row groups 256 bytes apart (one
// K=16 step of bf16 per 32-byte row).
__device__ __forceinline__ uint64_t sw32_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) | (static_cast<uint64_t>(1) << 16) |
         (static_cast<uint64_t>(256 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(6) << 61);
}

__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, int x, int y,
                                             const void* src) {
  asm volatile(
      "cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%1, %2}], [%3];" ::"l"(
          reinterpret_cast<uint64_t>(map)),
      "r"(x), "r"(y), "r"(smem_u32(src))
      : "memory");
}

// A[t] = [hi | lo | hi] of d_raw (backward record floats 0..23), B[k] = [hi | hi | lo] of
// hc_fn[k]; columns 72..127 zero. One thread per row, 16-byte stores.
__global__ void __launch_bounds__(256) pre_bwd_split_kernel(const float* __restrict__ brec,
                                                            const float* __restrict__ W,
                                                            uint16_t* __restrict__ A,
                                                            uint16_t* __restrict__ B, int64_t T,
                                                            int64_t K, int rec_stride) {
  pdl_wait();
  pdl_trigger();
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < T + K;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const bool is_a = r < T;
    const float* src = is_a ? brec + r * rec_stride : W + (r - T) * kMix;
    uint16_t* dst = is_a ? A + r * kDrKd : B + (r - T) * kDrKd;
    uint16_t hi[kMix], lo[kMix];
#pragma unroll
    for (int j = 0; j < kMix; ++j) {
      const float v = src[j];
      hi[j] = f32_to_bf16(v);
      lo[j] = f32_to_bf16(v - bf16_to_f32(hi[j]));
    }
    uint32_t row[64];  // 128 bf16
#pragma unroll
    for (int c = 0; c < 64; ++c) {
      uint16_t e[2];
#pragma unroll
      for (int u = 0; u < 2; ++u) {
        const int col = 2 * c + u;
        const int grp = col / kMix, j = col - grp * kMix;
        e[u] = col >= 3 * kMix ? 0
               : grp == 0       ? hi[j]
               : grp == 1       ? (is_a ? lo[j] : hi[j])
                                : (is_a ? hi[j] : lo[j]);
      }
      row[c] = static_cast<uint32_t>(e[0]) | (static_cast<uint32_t>(e[1]) << 16);
    }
#pragma unroll
    for (int q = 0; q < 16; ++q)
      reinterpret_cast<uint4*>(dst)[q] =
          make_uint4(row[4 * q], row[4 * q + 1], row[4 * q + 2], row[4 * q + 3]);
  }
}

struct DrArgs {
  const float* brec;
  float* dwp;  // d_hc_fn partials [nck * S][4H][24]
  int64_t T, H, ntt, nhc, W, nck;
  int rec_stride, S;
  int has_dy;  // 0: d_y absent (zero), no d_y tiles are loaded
};

// Item w of the flattened list: chunk ck of kDrwChunk token tiles (slowest), column block hc,
// token tile tt, stream i (fastest). The unit (ck, hc) is the run of items whose d_hc_fn products
// share a partial slice; u0, u1 are its first and last items.
struct DrwItem {
  int64_t hc, tt, i, ck, u0, u1;
};
__host__ __device__ __forceinline__ DrwItem drw_item(const DrArgs& a, int64_t w) {
  DrwItem r;
  const int64_t per_ck = a.nhc * kDrwChunk * 4;  // items of a full chunk
  r.ck = w / per_ck;
  const int64_t t0 = r.ck * kDrwChunk;           // the chunk's first token tile
  const int64_t ct = a.ntt - t0 < kDrwChunk ? a.ntt - t0 : kDrwChunk;
  const int64_t rem = w - r.ck * per_ck;
  r.hc = rem / (ct * 4);
  const int64_t rem2 = rem - r.hc * ct * 4;
  r.tt = t0 + (rem2 >> 2);
  r.i = rem2 & 3;
  r.u0 = r.ck * per_ck + r.hc * ct * 4;
  r.u1 = r.u0 + ct * 4 - 1;
  return r;
}

// MN-major, 128-byte swizzle: the next 64-element atom along M (or N) one 16 KB box on (leading
// byte offset), the next 8 tokens 1 KB on (stride byte offset).
__device__ __forceinline__ uint64_t drw_mn_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>(kDrAtom >> 4) << 16) | (static_cast<uint64_t>(1024 >> 4) << 32) |
         (static_cast<uint64_t>(1) << 46) | (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void drw_umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kDrwIdesc), "r"(accumulate)
      : "memory");
}

__global__ void __launch_bounds__(kDrThreads, 1)
    pre_bwd_drw_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                       const __grid_constant__ CUtensorMap tmA16, const __grid_constant__ CUtensorMap tmB16,
                       const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmDy,
                       const __grid_constant__ CUtensorMap tmDR, const DrArgs a) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* sA = smem + kDrOffA;
  uint8_t* sDy = smem + kDrOffDy;
  uint8_t* sB = smem + kDrOffB;
  uint8_t* sRr = smem + kDrOffR;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kDrOffBars);
  uint64_t* rfull = bars;          // [3] R tile landed
  uint64_t* rempty = bars + 3;     // [3] d_R stored from the slot (the store has read it)
  uint64_t* afull = bars + 6;      // [2] d_R accumulator ready (and the item's d_hc_fn MMAs done)
  uint64_t* aempty = bars + 8;     // [2] d_R accumulator read out (4 warps)
  uint64_t* dyfull = bars + 10;    // [2] d_y buffer landed
  uint64_t* dyempty = bars + 12;   // [2] d_y buffer's group finished (4 warps)
  uint64_t* abar = bars + 14;      // A landed
  uint64_t* adone = bars + 15;     // MMAs on the current A finished
  uint64_t* done = bars + 16;
  uint64_t* bfull = bars + 17;     // [2] B landed
  uint64_t* bempty = bars + 19;    // [2] MMAs on B finished
  uint64_t* drready = bars + 21;   // [3] d_R tile of an R slot written (4 warps)
  uint64_t* wfull = bars + 24;     // d_hc_fn accumulators of a piece complete
  uint64_t* wempty = bars + 25;    // d_hc_fn accumulators read out (4 warps)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 26);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t lo = blockIdx.x * a.W / P, hi = (blockIdx.x + 1) * a.W / P;

  if (threadIdx.x == 0) {
    for (int r = 0; r < kDrRSlots; ++r) {
      mbar_init(&rfull[r], 1);
      mbar_init(&rempty[r], 1);
      mbar_init(&drready[r], 4);
    }
    for (int b = 0; b < kDrBSlots; ++b) {
      mbar_init(&bfull[b], 1);
      mbar_init(&bempty[b], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&afull[b], 1);
      mbar_init(&aempty[b], 4);
      mbar_init(&dyfull[b], 1);
      mbar_init(&dyempty[b], 4);
    }
    mbar_init(abar, 1);
    mbar_init(adone, 1);
    mbar_init(done, 1);
    mbar_init(wfull, 1);
    mbar_init(wempty, 4);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kDrTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the records, the split operands and d_R's previous readers are done

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (R, B, d_y)
    if (lane == 0) {
      int64_t it = 0, nbl = 0, ng = 0, cur_g = -1;
      bool ok = true;
      for (int64_t w = lo; w < hi && ok; ++w) {
        const DrwItem d = drw_item(a, w);
        const int64_t g = w >> 2;
        const int y = static_cast<int>(d.tt * kDrM);
        if (a.has_dy && g != cur_g) {
          const int gb = static_cast<int>(ng & 1);
          if (ng >= 2 &&
              !mbar_wait(&dyempty[gb], static_cast<uint32_t>((ng - 2) >> 1) & 1u, 91)) {
            ok = false;
            break;
          }
          uint8_t* dd = sDy + gb * kDrTile;
          mbar_arrive_expect_tx(&dyfull[gb], kDrTile);
          tma_load_2d(dd, &tmDy, static_cast<int>(d.hc * kDrN), y, &dyfull[gb]);
          tma_load_2d(dd + kDrAtom, &tmDy, static_cast<int>(d.hc * kDrN + 64), y, &dyfull[gb]);
          ++ng;
          cur_g = g;
        }
        const int k0 = static_cast<int>(d.i * a.H + d.hc * kDrN);
        // R first (the HBM stream; the ring slot is free once the item three back is stored),
        // then B (free once the MMAs two items back have read it).
        const int rs = static_cast<int>(it % kDrRSlots);
        if (it >= kDrRSlots &&
            !mbar_wait(&rempty[rs], static_cast<uint32_t>((it - kDrRSlots) / kDrRSlots) & 1u, 92)) {
          ok = false;
          break;
        }
        uint8_t* rt = sRr + rs * kDrTile;
        mbar_arrive_expect_tx(&rfull[rs], kDrTile);
        tma_load_2d(rt, &tmR, k0, y, &rfull[rs]);
        tma_load_2d(rt + kDrAtom, &tmR, k0 + 64, y, &rfull[rs]);
        ++it;
        const int bs = static_cast<int>(nbl % kDrBSlots);
        if (nbl >= kDrBSlots &&
            !mbar_wait(&bempty[bs], static_cast<uint32_t>((nbl - kDrBSlots) / kDrBSlots) & 1u, 92)) {
          ok = false;
          break;
        }
        uint8_t* bt = sB + bs * kDrOpTile;
        mbar_arrive_expect_tx(&bfull[bs], kDrOpTile);
        tma_load_2d(bt, &tmB, 0, k0, &bfull[bs]);
        tma_load_2d(bt + kDrAtom, &tmB16, 64, k0, &bfull[bs]);
        ++nbl;
      }
      // Do not leave while copies into shared memory are in flight (every issued load completes
      // its barrier; waiting on the last phases of each is enough).
      if (!ok) {
        for (int64_t k = it - kDrRSlots; k < it; ++k)
          if (k >= 0)
            mbar_wait(&rfull[k % kDrRSlots], static_cast<uint32_t>(k / kDrRSlots) & 1u, 93);
        for (int64_t k = nbl - kDrBSlots; k < nbl; ++k)
          if (k >= 0)
            mbar_wait(&bfull[k % kDrBSlots], static_cast<uint32_t>(k / kDrBSlots) & 1u, 93);
        if (ng > 0) mbar_wait(&dyfull[(ng - 1) & 1], static_cast<uint32_t>((ng - 1) >> 1) & 1u, 93);
        if (ng > 1) mbar_wait(&dyfull[(ng - 2) & 1], static_cast<uint32_t>((ng - 2) >> 1) & 1u, 93);
      }
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (+ A loads)
    if (lane == 0) {
      int64_t it = 0, na_issued = 0, na = 0, nad = 0, cur_tt = -1, pc = 0, cur_u0 = -1;
      uint32_t started = 0;  // streams whose d_hc_fn accumulator this piece has begun
      bool ok = true;
      auto load_a = [&](int64_t tt) {
        mbar_arrive_expect_tx(abar, kDrOpTile);
        tma_load_2d(sA, &tmA, 0, static_cast<int>(tt * kDrM), abar);
        tma_load_2d(sA + kDrAtom, &tmA16, 64, static_cast<int>(tt * kDrM), abar);
        ++na_issued;
      };
      if (lo < hi) load_a(drw_item(a, lo).tt);
      for (int64_t w = lo; w < hi && ok; ++w) {
        const DrwItem d = drw_item(a, w);
        if (d.tt != cur_tt) {
          if (!mbar_wait(abar, static_cast<uint32_t>(na) & 1u, 95)) {
            ok = false;
            break;
          }
          ++na;
          cur_tt = d.tt;
        }
        if (d.u0 != cur_u0) {  // a new piece: the previous piece's accumulators have been read
          if (pc > 0 && !mbar_wait(wempty, static_cast<uint32_t>(pc - 1) & 1u, 103)) {
            ok = false;
            break;
          }
          started = 0;
          cur_u0 = d.u0;
          ++pc;
        }
        const int rs = static_cast<int>(it % kDrRSlots);
        const int b = static_cast<int>(it & 1);
        const int bs = static_cast<int>(it % kDrBSlots);
        if (!mbar_wait(&rfull[rs], static_cast<uint32_t>(it / kDrRSlots) & 1u, 104)) {
          ok = false;
          break;
        }
        if (!mbar_wait(&bfull[bs], static_cast<uint32_t>(it / kDrBSlots) & 1u, 96)) {
          ok = false;
          break;
        }
        if (it >= 2 && !mbar_wait(&aempty[b], static_cast<uint32_t>((it - 2) >> 1) & 1u, 97)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t aaddr = smem_u32(sA);
        const uint32_t baddr = smem_u32(sB + bs * kDrOpTile);
        const uint32_t raddr = smem_u32(sRr + rs * kDrTile);
        // d_hc_fn of stream i: D_i[k][n] += sum_t R[t][k] A[t][n] over the tile's 128 tokens
        // (A = R MN-major, M = 128 columns k; B = the A tile's first 64 split columns, MN-major).
        const uint32_t dw = tmem + static_cast<uint32_t>(kDrwCol0 + kDrwN * d.i);
        const uint32_t first = (started >> d.i) & 1u;
#pragma unroll
        for (int k = 0; k < kDrM / 16; ++k)  // 16 tokens: +2 KB in both operands
          drw_umma(dw, drw_mn_desc(raddr) + 128 * k, drw_mn_desc(aaddr) + 128 * k,
                   (first != 0u || k > 0) ? 1u : 0u);
        started |= 1u << d.i;
        // d_R's contraction.
        const uint32_t dt = tmem + static_cast<uint32_t>(b * kDrN);
#pragma unroll
        for (int k = 0; k < 4; ++k)  // split columns 0..63: +32 bytes along the row per step
          dr_umma(dt, sw128_desc(aaddr) + 2 * k, sw128_desc(baddr) + 2 * k, k > 0 ? 1u : 0u);
        dr_umma(dt, sw32_desc(aaddr + kDrAtom), sw32_desc(baddr + kDrAtom), 1u);  // 64..79
        umma_commit(&bempty[bs]);  // B read: the slot may take a later item's B
        umma_commit(&afull[b]);    // also covers the d_hc_fn MMAs that read the R slot
        ++it;
        if (w == d.u1 || w + 1 == hi) umma_commit(wfull);  // the piece's accumulators
        // The next item needs another token tile: reload A once these MMAs have read it.
        if (w + 1 < hi) {
          const int64_t ntt = drw_item(a, w + 1).tt;
          if (ntt != d.tt) {
            umma_commit(adone);
            if (!mbar_wait(adone, static_cast<uint32_t>(nad) & 1u, 94)) {
              ok = false;
              break;
            }
            ++nad;
            load_a(ntt);
          }
        }
      }
      // Do not leave while an A load is in flight.
      if (!ok && na_issued > na) mbar_wait(abar, static_cast<uint32_t>(na) & 1u, 93);
      umma_commit(done);  // every issued MMA has finished before TMEM is released
      mbar_wait(done, 0, 98);
    }
  } else if (warp < 6) {
    // ------------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quarter
    const int row = q * 32 + lane;
    int64_t it = 0, ng = 0, cur_g = -1, pc = 0;
    int gb = 0;
    uint32_t gph = 0;
    for (int64_t w = lo; w < hi; ++w) {
      const DrwItem d = drw_item(a, w);
      const int64_t g = w >> 2;
      if (g != cur_g) {
        if (cur_g >= 0) {  // this warp is done with the previous group's d_y buffer
          __syncwarp();
          if (lane == 0) mbar_arrive(&dyempty[gb]);
        }
        gb = static_cast<int>(ng & 1);
        gph = static_cast<uint32_t>(ng >> 1) & 1u;
        ++ng;
        cur_g = g;
      }
      const int rs = static_cast<int>(it % kDrRSlots);
      const int b = static_cast<int>(it & 1);
      bool ok = __all_sync(
          0xffffffffu,
          mbar_wait(&rfull[rs], static_cast<uint32_t>(it / kDrRSlots) & 1u, 99));
      ok = ok && (!a.has_dy || __all_sync(0xffffffffu, mbar_wait(&dyfull[gb], gph, 100)));
      ok = ok && __all_sync(0xffffffffu,
                            mbar_wait(&afull[b], static_cast<uint32_t>(it >> 1) & 1u, 101));
      // The four warps agree on going on (a stop keeps the named-barrier sequence matched).
      if (named_bar_or(1, 128, !ok)) break;
      tc_fence_after();
      const int64_t tok = d.tt * kDrM + row;
      float dss2 = 0.f, pi = 0.f;
      if (tok < a.T) {
        dss2 = 2.0f * __ldg(a.brec + tok * a.rec_stride + 24);
        pi = __ldg(a.brec + tok * a.rec_stride + 25 + d.i);
      }
      uint8_t* sR = sRr + rs * kDrTile;
      const uint8_t* sY = sDy + gb * kDrTile;
      const uint32_t tbase =
          tmem + static_cast<uint32_t>(b * kDrN) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll 1
      for (int half = 0; half < 2; ++half) {
        uint32_t acc[2][32];
        tmem_ld32(tbase + half * 64, acc[0]);
        tmem_ld32(tbase + half * 64 + 32, acc[1]);
        tmem_wait_ld();
#pragma unroll
        for (int hq = 0; hq < 2; ++hq) {
          const int cq = half * 2 + hq;
          const int atom = cq >> 1;
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            // 16-byte chunk c of the row's 128-byte swizzled line sits at chunk c ^ (row & 7).
            const int c = (cq & 1) * 4 + u;
            const int off = atom * kDrAtom + row * 128 + ((c ^ (row & 7)) << 4);
            const uint4 rv = *reinterpret_cast<const uint4*>(sR + off);
            const uint4 yv =
                a.has_dy ? *reinterpret_cast<const uint4*>(sY + off) : make_uint4(0u, 0u, 0u, 0u);
            const uint32_t r4[4] = {rv.x, rv.y, rv.z, rv.w};
            const uint32_t y4[4] = {yv.x, yv.y, yv.z, yv.w};
            uint32_t o[4];
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float a0 = __uint_as_float(acc[hq][8 * u + 2 * e]);
              const float a1 = __uint_as_float(acc[hq][8 * u + 2 * e + 1]);
              o[e] = pack_bf16x2(fmaf(pi, bf16_lo(y4[e]), fmaf(dss2, bf16_lo(r4[e]), a0)),
                                 fmaf(pi, bf16_hi(y4[e]), fmaf(dss2, bf16_hi(r4[e]), a1)));
            }
            *reinterpret_cast<uint4*>(sR + off) = make_uint4(o[0], o[1], o[2], o[3]);
          }
        }
      }
      tc_fence_before();
      // The rows are written: the accumulator goes back to the MMA warp, and the d_R tile (in R's
      // slot) to the storer, with the generic-proxy writes made visible to the TMA engine.
      asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&aempty[b]);
        mbar_arrive(&drready[rs]);
      }
      ++it;
      if (w != d.u1 && w + 1 != hi) continue;
      // ---- the piece's end: d_hc_fn partials of its four streams, thread = column k of the
      // block (TMEM lane), into slot (this CTA's rank among the unit's CTAs) of chunk d.ck.
      ok = __all_sync(0xffffffffu, mbar_wait(wfull, static_cast<uint32_t>(pc) & 1u, 105));
      if (named_bar_or(1, 128, !ok)) break;
      tc_fence_after();
      const int64_t ps = lo > d.u0 ? lo : d.u0;
      const int64_t n = w - ps + 1;  // the piece's items ps..w
      const int64_t slot = static_cast<int64_t>(blockIdx.x) - tc_first_cta(d.u0, P, a.W);
      const int64_t K = 4 * a.H;
      for (int s = 0; s < 4; ++s) {
        // Stream s has an item in the piece iff its first position after ps is within n.
        const bool present = ((s - static_cast<int>(ps & 3)) & 3) < n;
        float v[kMix];
        if (present) {
          uint32_t dd[3][16];
          const uint32_t wb = tmem + static_cast<uint32_t>(kDrwCol0 + kDrwN * s) +
                              (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
          for (int cc = 0; cc < 3; ++cc) tmem_ld16(wb + cc * 16, dd[cc]);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < kMix; ++j)  // columns j: R.hi(d_raw_j), 24 + j: R.lo(d_raw_j)
            v[j] = __uint_as_float(dd[(kMix + j) / 16][(kMix + j) % 16]) +
                   __uint_as_float(dd[j / 16][j % 16]);
        } else {
#pragma unroll
          for (int j = 0; j < kMix; ++j) v[j] = 0.f;
        }
        const int64_t k = s * a.H + d.hc * kDrN + row;
        float4* dst = reinterpret_cast<float4*>(a.dwp + ((d.ck * a.S + slot) * K + k) * kMix);
#pragma unroll
        for (int w4 = 0; w4 < kMix / 4; ++w4)
          dst[w4] = make_float4(v[4 * w4], v[4 * w4 + 1], v[4 * w4 + 2], v[4 * w4 + 3]);
        if (w == d.u1) {  // the unit's last piece: zero its unused slots
          for (int64_t sl = slot + 1; sl < a.S; ++sl) {
            float4* z = reinterpret_cast<float4*>(a.dwp + ((d.ck * a.S + sl) * K + k) * kMix);
#pragma unroll
            for (int w4 = 0; w4 < kMix / 4; ++w4) z[w4] = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(wempty);
      ++pc;
    }
  } else if (warp == 6) {
    // ------------------------------------------------------------------ d_R storer
    if (lane == 0) {
      int64_t it = 0;
      for (int64_t w = lo; w < hi; ++w, ++it) {
        const DrwItem d = drw_item(a, w);
        const int rs = static_cast<int>(it % kDrRSlots);
        if (!mbar_wait(&drready[rs], static_cast<uint32_t>(it / kDrRSlots) & 1u, 102)) break;
        const uint8_t* sR = sRr + rs * kDrTile;
        const int x = static_cast<int>(d.i * a.H + d.hc * kDrN);
        const int y = static_cast<int>(d.tt * kDrM);
        tma_store_2d(&tmDR, x, y, sR);
        tma_store_2d(&tmDR, x + 64, y, sR + kDrAtom);
        asm volatile("cp.async.bulk.commit_group;" ::: "memory");
        asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // the slot has been read
        mbar_arrive(&rempty[rs]);
      }
      asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");  // stores complete before exit
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kDrTmemCols)
                 : "memory");
  }
}

// ------------------------------------------------------------------------------ d_hc_fn
//
// d_hc_fn[k][j] = sum_t R[t][k] d_raw[t][j]: a contraction over tokens. The MMA's M is 128 features
// k, its K the tokens, so the A operand is R itself read MN-major: a TMA box [64 tokens x 64
// features] of R lands as 64 lines of 128 bytes (one token each, features contiguous) with the
// 128-byte swizzle, which is the MN-major swizzled atom (64 features x 8 tokens, 1 KB); the two
// boxes of a 128-feature tile are the two atoms along M. B = [hi(d_raw) | lo(d_raw)] transposed,
// [48][tokens] bf16 (K-major), so each product is hi.R + lo.R, exact in fp32 (R is exact in bf16;
// hi + lo leaves below 2^-16 of d_raw).
//
// pre_bwd_dw_kernel_tc: persistent, two CTAs per SM; the (feature tile, 64-token block) units,
// tile-major, cut into equal contiguous ranges; a range covers pieces (tile, token interval) whose
// rank among the tile's pieces is their slot. Warp 0: TMA of both R boxes and the B block per
// stage (4 stages of 22 KB); warp 1: four M=128 N=48 K=16 MMAs per block into one of two TMEM
// accumulators, restarted every 16 blocks (1024 tokens: short fp32 chains); warps 2-5: each
// finished sub-piece's accumulator (tcgen05.ld) added, as hi + lo, into registers in order; at
// the piece's end the thread of feature k writes the partial [slot][k][24]. The CTA holding a
// tile's last piece zero-fills the tile's unused slots; pre_bwd_dw_sum_kernel adds the slots in
// order.

constexpr int kWtM = 128;
constexpr int kWtN = 48;
constexpr int kWtTok = 64;                         // tokens per block
constexpr int kWtABytes = 2 * kWtTok * 128;        // two [64 x 64] boxes of R: 16 KB
constexpr int kWtBBytes = kWtN * 128;              // [48 x 64 tokens]: 6 KB
constexpr int kWtStageBytes = kWtABytes + kWtBBytes;  // 22528 = 22 x 1024
constexpr int kWtStages = 4;
// Slack after the stages: an MMA reading through a misread descriptor stride stays inside the
// allocation (the tile spans at most 16 KB from its base whatever the strides' roles).
constexpr int kWtSlack = 16384;
constexpr int kWtOffBars = kWtStages * kWtStageBytes + kWtSlack;
constexpr int kWtSmem = 1024 + kWtOffBars + 256;
constexpr int kWtThreads = 192;
constexpr int kWtTmemCols = 128;                   // two accumulators of 48 columns (0, 64)
constexpr int kWtSubBlocks = 16;
constexpr int kWtMinUnits = 8;
// kind::f16, D fp32, A and B bf16, A MN-major (bit 15), B K-major, N = 48, M = 128.
constexpr uint32_t kWtIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (1u << 15) |
                              (static_cast<uint32_t>(kWtN >> 3) << 17) |
                              (static_cast<uint32_t>(kWtM >> 4) << 24);

// MN-major, 128-byte swizzle: the second 64-feature atom 8 KB on (leading byte offset), the next
// 8 tokens 1 KB on (stride byte offset).
__device__ __forceinline__ uint64_t sw128_mn_desc(uint32_t saddr) {
  return static_cast<uint64_t>((saddr >> 4) & 0x3FFFu) |
         (static_cast<uint64_t>(kWtTok * 128 >> 4) << 16) |
         (static_cast<uint64_t>(1024 >> 4) << 32) | (static_cast<uint64_t>(1) << 46) |
         (static_cast<uint64_t>(2) << 61);
}

__device__ __forceinline__ void wt_umma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                        uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(kWtIdesc), "r"(accumulate)
      : "memory");
}

struct WtPlan {
  int64_t nk, NB, Tp, W, P, S;
};

static WtPlan wt_plan(int64_t T, int64_t H, int64_t sms) {
  WtPlan p;
  p.nk = 4 * H / kWtM;
  p.NB = (T + kWtTok - 1) / kWtTok;
  p.Tp = p.NB * kWtTok;
  p.W = p.nk * p.NB;
  p.P = 2 * sms;
  if (p.P > 2 * 148) p.P = 2 * 148;
  if (p.P > p.W / kWtMinUnits) p.P = p.W / kWtMinUnits;
  if (p.P < 1) p.P = 1;
  p.S = p.NB * p.P / p.W + 2;  // pieces one tile meets at most
  if (p.S > p.P) p.S = p.P;
  return p;
}

bool pre_bwd_dw_tc_supported(int64_t T, int64_t H) {
  return T >= 1 && H >= 32 && (4 * H) % kWtM == 0 && (T + kWtTok - 1) / kWtTok <= (1 << 24);
}

size_t pre_bwd_dw_tc_workspace_bytes(int64_t T, int64_t H) {
  if (!pre_bwd_dw_tc_supported(T, H)) return 0;
  const WtPlan p = wt_plan(T, H, 148);
  auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
  return up(static_cast<size_t>(kWtN) * p.Tp * 2) +
         up(static_cast<size_t>(p.S) * 4 * H * kMix * 4);
}

// Bt[n][t] = hi(d_raw[t][n]) for n < 24, lo(...) for 24 <= n < 48 (zero for t >= T): consecutive
// threads take consecutive tokens, so each row's stores coalesce.
__global__ void __launch_bounds__(256) pre_bwd_bt_kernel(const float* __restrict__ brec,
                                                         uint16_t* __restrict__ Bt, int64_t T,
                                                         int64_t Tp, int rec_stride) {
  pdl_wait();
  pdl_trigger();
  for (int64_t t = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; t < Tp;
       t += static_cast<int64_t>(gridDim.x) * blockDim.x) {
#pragma unroll 4
    for (int j = 0; j < kMix; ++j) {
      const float v = t < T ? brec[t * rec_stride + j] : 0.f;
      const uint16_t hi = f32_to_bf16(v);
      Bt[j * Tp + t] = hi;
      Bt[(kMix + j) * Tp + t] = f32_to_bf16(v - bf16_to_f32(hi));
    }
  }
}

__global__ void __launch_bounds__(kWtThreads, 2) pre_bwd_dw_kernel_tc(
    const __grid_constant__ CUtensorMap tmR, const __grid_constant__ CUtensorMap tmBt,
    float* __restrict__ dwp, int64_t K, int64_t NB, int64_t W, int S) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + kWtOffBars);
  uint64_t* full = bars;                    // [4]
  uint64_t* empty = bars + kWtStages;       // [4] MMA commit
  uint64_t* afull = bars + 2 * kWtStages;   // [2]
  uint64_t* aempty = afull + 2;             // [2] 4 warps
  uint64_t* done = aempty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(done + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t lo = c * W / P, hi = (c + 1) * W / P;

  if (threadIdx.x == 0) {
    for (int st = 0; st < kWtStages; ++st) {
      mbar_init(&full[st], 1);
      mbar_init(&empty[st], 1);
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
                 "r"(kWtTmemCols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();

  if (warp == 0) {
    if (lane == 0) {
      int64_t n = 0;
      bool ok = true;
      for (int64_t u = lo; u < hi; ++u, ++n) {
        const int64_t kt = u / NB;
        const int tb = static_cast<int>(u - kt * NB);
        const int st = static_cast<int>(n % kWtStages);
        if (n >= kWtStages &&
            !mbar_wait(&empty[st], static_cast<uint32_t>((n / kWtStages) - 1) & 1u, 110)) {
          ok = false;
          break;
        }
        uint8_t* sa = smem + st * kWtStageBytes;
        mbar_arrive_expect_tx(&full[st], kWtStageBytes);
        tma_load_2d(sa, &tmR, static_cast<int>(kt * kWtM), tb * kWtTok, &full[st]);
        tma_load_2d(sa + kWtTok * 128, &tmR, static_cast<int>(kt * kWtM + 64), tb * kWtTok,
                    &full[st]);
        tma_load_2d(sa + kWtABytes, &tmBt, tb * kWtTok, 0, &full[st]);
      }
      if (!ok) {  // do not leave while copies into shared memory are in flight
        for (int64_t i = n - kWtStages; i < n; ++i)
          if (i >= 0)
            mbar_wait(&full[i % kWtStages], static_cast<uint32_t>(i / kWtStages) & 1u, 111);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t n = 0, sp = 0;
      bool ok = true;
      uint32_t dt = tmem;
      for (int64_t u = lo; u < hi && ok;) {
        const int64_t kt = u / NB;
        const int64_t tbs = u - kt * NB;
        const int64_t tbe = min(NB, tbs + (hi - u));
        for (int64_t tb = tbs; tb < tbe; ++tb, ++n) {
          const int ks = static_cast<int>((tb - tbs) % kWtSubBlocks);
          if (ks == 0) {
            const int b = static_cast<int>(sp & 1);
            if (sp >= 2 &&
                !mbar_wait(&aempty[b], static_cast<uint32_t>((sp >> 1) - 1) & 1u, 112)) {
              ok = false;
              break;
            }
            tc_fence_after();
            dt = tmem + static_cast<uint32_t>(b * 64);
          }
          const int st = static_cast<int>(n % kWtStages);
          if (!mbar_wait(&full[st], static_cast<uint32_t>(n / kWtStages) & 1u, 113)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = smem_u32(smem + st * kWtStageBytes);
          const uint64_t adesc = sw128_mn_desc(sa);
          const uint64_t bdesc = sw128_desc(sa + kWtABytes);
#pragma unroll
          for (int k = 0; k < kWtTok / 16; ++k)  // 16 tokens: +2 KB of A, +32 bytes of B's rows
            wt_umma(dt, adesc + 128 * k, bdesc + 2 * k, (ks > 0 || k > 0) ? 1u : 0u);
          umma_commit(&empty[st]);
          if (tb + 1 == tbe || ks + 1 == kWtSubBlocks) {
            umma_commit(&afull[sp & 1]);
            ++sp;
          }
        }
        u += tbe - tbs;
      }
      umma_commit(done);
      mbar_wait(done, 0, 114);
    }
  } else {
    // Warps 2..5: TMEM lane quarter q holds features 32q .. 32q + 31 of the tile.
    const int q = warp & 3;
    const int row = q * 32 + lane;
    int64_t sp = 0;
    bool ok = true;
    for (int64_t u = lo; u < hi && ok;) {
      const int64_t kt = u / NB;
      const int64_t tbs = u - kt * NB;
      const int64_t tbe = min(NB, tbs + (hi - u));
      float racc[kMix];
#pragma unroll
      for (int j = 0; j < kMix; ++j) racc[j] = 0.f;
      for (int64_t b0 = tbs; b0 < tbe; b0 += kWtSubBlocks, ++sp) {
        const int b = static_cast<int>(sp & 1);
        if (!__all_sync(0xffffffffu,
                        mbar_wait(&afull[b], static_cast<uint32_t>(sp >> 1) & 1u, 115))) {
          ok = false;
          break;
        }
        tc_fence_after();
        uint32_t d[3][16];
        const uint32_t tbase =
            tmem + static_cast<uint32_t>(b * 64) + (static_cast<uint32_t>(q * 32) << 16);
#pragma unroll
        for (int cc = 0; cc < 3; ++cc) tmem_ld16(tbase + cc * 16, d[cc]);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < kMix; ++j) {
          const float h = __uint_as_float(d[j / 16][j % 16]);
          const float l = __uint_as_float(d[(kMix + j) / 16][(kMix + j) % 16]);
          racc[j] += l + h;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&aempty[b]);
      }
      if (!ok) break;
      const int64_t slot = c - tc_first_cta(kt * NB, P, W);
      const int64_t k = kt * kWtM + row;
      float4* dst = reinterpret_cast<float4*>(dwp + (slot * K + k) * kMix);
#pragma unroll
      for (int w4 = 0; w4 < kMix / 4; ++w4)
        dst[w4] = make_float4(racc[4 * w4], racc[4 * w4 + 1], racc[4 * w4 + 2], racc[4 * w4 + 3]);
      if (tbe == NB) {  // the tile's last piece: zero its unused slots
        for (int64_t sl = slot + 1; sl < S; ++sl) {
          float4* z = reinterpret_cast<float4*>(dwp + (sl * K + k) * kMix);
#pragma unroll
          for (int w4 = 0; w4 < kMix / 4; ++w4) z[w4] = make_float4(0.f, 0.f, 0.f, 0.f);
        }
      }
      u += tbe - tbs;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kWtTmemCols)
                 : "memory");
  }
}

// d_hc_fn on tensor cores: Bt, the partials, their in-order sum. Returns 0, a negative MHC_ERR_*
// code, or 1 when this form cannot run (nothing launched).
int launch_pre_bwd_dw_tc(const uint16_t* R, const float* brec, int rec_stride, float* dW,
                         void* ws, int64_t T, int64_t H, cudaStream_t s) {
  if (!pre_bwd_dw_tc_supported(T, H) || !aligned16(R) || !aligned16(ws)) return 1;
  if (!ensure_smem_limit(reinterpret_cast<const void*>(pre_bwd_dw_kernel_tc), kWtSmem)) return 1;
  const int64_t K = 4 * H;
  const WtPlan plan = wt_plan(T, H, device_sm_count());
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  uint16_t* Bt = reinterpret_cast<uint16_t*>(w8);
  float* dwp = reinterpret_cast<float*>(
      w8 + (static_cast<size_t>(kWtN) * plan.Tp * 2 + 1023) / 1024 * 1024);
  CUtensorMap mR, mBt;
  if (!make_map(&mR, R, K, T, kWtTok) || !make_map(&mBt, Bt, plan.Tp, kWtN, kWtN)) return -4;
  int64_t nb = (plan.Tp + 255) / 256;
  if (nb > 148 * 8) nb = 148 * 8;
  if (launch_pdl(pre_bwd_bt_kernel, dim3(static_cast<unsigned>(nb)), dim3(256), 0, s, brec, Bt, T,
                 plan.Tp, rec_stride) != cudaSuccess)
    return -4;
  if (launch_pdl(pre_bwd_dw_kernel_tc, dim3(static_cast<unsigned>(plan.P)), dim3(kWtThreads),
                 static_cast<size_t>(kWtSmem), s, mR, mBt, dwp, K, plan.NB, plan.W,
                 static_cast<int>(plan.S)) != cudaSuccess)
    return -4;
  int64_t sb = (K * kMix + 255) / 256;
  if (sb > 148 * 8) sb = 148 * 8;
  if (launch_pdl(pre_bwd_dw_sum_kernel, dim3(static_cast<unsigned>(sb)), dim3(256), 0, s,
                 static_cast<const float*>(dwp), dW, K * kMix, static_cast<int>(plan.S)) !=
      cudaSuccess)
    return -4;
  note_launches(3);
  return 0;
}

// d_R and d_hc_fn on tensor cores: the split operands, the fused kernel, the partials' in-order
// sum. Returns 0, a negative MHC_ERR_* code, or 1 when this form cannot run (nothing launched).
int launch_pre_bwd_dr_tc(const uint16_t* R, const uint16_t* dy, const float* hc_fn,
                         const float* brec, int rec_stride, uint16_t* dR, float* dW, void* ws,
                         int64_t T, int64_t H, cudaStream_t s) {
  if (!pre_bwd_dr_tc_supported(T, H) || !aligned16(R) || (dy != nullptr && !aligned16(dy)) ||
      !aligned16(dR) || !aligned16(ws))
    return 1;
  if (!ensure_smem_limit(reinterpret_cast<const void*>(pre_bwd_drw_kernel), kDrSmem)) return 1;
  const int64_t K = 4 * H;
  const DrPlan plan = dr_plan(T, H, device_sm_count());
  auto up = [](size_t v) { return (v + 1023) / 1024 * 1024; };
  uint8_t* w8 = static_cast<uint8_t*>(ws);
  uint16_t* A = reinterpret_cast<uint16_t*>(w8);
  uint16_t* B = reinterpret_cast<uint16_t*>(w8 + up(static_cast<size_t>(T) * kDrKd * 2));
  float* dwp = reinterpret_cast<float*>(w8 + up(static_cast<size_t>(T) * kDrKd * 2) +
                                        up(static_cast<size_t>(K) * kDrKd * 2));
  CUtensorMap mA, mB, mA16, mB16, mR, mDy, mDR;
  // [rows x 16] boxes of columns 64..79, 32-byte swizzle.
  auto narrow_map = [](CUtensorMap* m, const void* base, int64_t rows) {
    EncodeTiledFn fn = encode_tiled();
    if (!fn) return false;
    const cuuint64_t dims[2] = {static_cast<cuuint64_t>(kDrKd), static_cast<cuuint64_t>(rows)};
    const cuuint64_t strides[1] = {static_cast<cuuint64_t>(kDrKd) * 2};
    const cuuint32_t box[2] = {16, 128};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
              estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B,
              CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
  };
  if (!make_map(&mA, A, kDrKd, T, kDrM) || !make_map(&mB, B, kDrKd, K, kDrN) ||
      !narrow_map(&mA16, A, T) || !narrow_map(&mB16, B, K) ||
      !make_map(&mR, R, K, T, kDrM) || !make_map(&mDR, dR, K, T, kDrM))
    return -4;
  if (dy == nullptr)
    mDy = mR;  // not read: no d_y tile is loaded
  else if (!make_map(&mDy, dy, H, T, kDrM))
    return -4;
  int64_t nb = (T + K + 255) / 256;
  if (nb > 148 * 8) nb = 148 * 8;
  if (launch_pdl(pre_bwd_split_kernel, dim3(static_cast<unsigned>(nb)), dim3(256), 0, s, brec,
                 hc_fn, A, B, T, K, rec_stride) != cudaSuccess)
    return -4;
  DrArgs da;
  da.brec = brec;
  da.dwp = dwp;
  da.T = T;
  da.H = H;
  da.ntt = plan.ntt;
  da.nhc = plan.nhc;
  da.W = plan.W;
  da.nck = plan.nck;
  da.rec_stride = rec_stride;
  da.S = static_cast<int>(plan.S);
  da.has_dy = dy != nullptr ? 1 : 0;
  if (launch_pdl(pre_bwd_drw_kernel, dim3(static_cast<unsigned>(plan.P)), dim3(kDrThreads),
                 static_cast<size_t>(kDrSmem), s, mA, mB, mA16, mB16, mR, mDy, mDR, da) !=
      cudaSuccess)
    return -4;
  int64_t sb = (K * kMix + 255) / 256;
  if (sb > 148 * 8) sb = 148 * 8;
  if (launch_pdl(pre_bwd_dw_sum_kernel, dim3(static_cast<unsigned>(sb)), dim3(256), 0, s,
                 static_cast<const float*>(dwp), dW, K * kMix,
                 static_cast<int>(plan.nck * plan.S)) != cudaSuccess)
    return -4;
  note_launches(3);
  return 0;
}

}  // namespace mhc
