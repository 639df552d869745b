// Post-map fused with the next site's projection partials.
//
// Pre and post alternate along the layer stack ("FlashInfer mHC module deep dive" §1: the two
// phases of every layer; glm5next_mhc.rs: the streams glm_hc_post writes are the next site's
// residual). The next site's pre-map starts by projecting the new residual row (out, flattened
// k = n*H + h) through its hc_fn and summing its squares; both are sums over k, so they can be
// formed while out is produced, as split partials that mhc_pre_big_fuse ("FlashInfer mHC module
// deep dive" §3.1-3.3: dot_mix / sqrsum with num_splits) then reduces. The next pre-map reads out
// once (aggregate) instead of twice.
//
// out[t][n][h] = bf16_rn(x[t][h]*post[t][n] + sum_o R[t][o][h]*comb[t][o][n]) with exactly the
// arithmetic of the post-map kernels (so out is bitwise equal to mhc_post's); then per token
// dot_mix[s][t][j] = sum_{k in split s} out_flat[t][k] * hc_fn_next[k][j] and
// sqrsum[s][t] = sum_{k in split s} out_flat[t][k]^2, over the bf16 values of out.
//
// Persistent kernel, one CTA per SM. Work: token tiles of 128; a tile's 64-column blocks are
// grouped into at most 16 chunks of L blocks, and a chunk's rank in its tile is its split; the
// tile-major list of chunks is cut into equal contiguous ranges, one per CTA. Roles:
//   warp 0      TMA: the 4 Bw blocks (k = n*H + h0, n = 0..3, [80 x 64] each, 128-byte swizzle)
//               of a column block into a 2-stage ring.
//   warp 1      tcgen05.mma M=128 N=80 K=16: for each column block, 4 streams x 4 K-steps into
//               the piece's TMEM accumulator (two, alternating between pieces).
//   warps 2-9   the post-map: 8 lanes per token row (one 16-byte chunk each), four tokens per
//               thread. The four R streams arrive one block ahead by 16-byte asynchronous copies
//               straight into the MMA A operand tiles (128-byte swizzled rows), x into registers;
//               out is computed in place there (it becomes the A operand) and stored to global
//               with 16-byte stores; sum of squares of the rounded outputs. After a piece they read the
//               accumulator (tcgen05.ld) and, with the sums of squares, write the split partials.
// Requires H % 8 == 0 and 16-byte aligned x, R, out, post, comb, dot_mix. out may be R.
#include <cuda.h>

#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

constexpr int kPpM = 128;                          // tokens per tile (MMA M)
constexpr int kPpHB = 64;                          // columns per block (one swizzled row)
constexpr int kPpABytes = kPpM * kPpHB * 2;        // 16384: one stream's A tile
constexpr int kPpBBytes = 80 * kPpHB * 2;          // 10240: one Bw block
constexpr int kPpAStage = 4 * kPpABytes;           // 65536
constexpr int kPpBStage = 4 * kPpBBytes;           // 40960
constexpr int kPpStages = 2;
constexpr int kPpXWarps = 8;                       // post-map warps (2..9)
constexpr int kPpEpiWarps = 8;                     // of them, those that read TMEM (2..9)
constexpr int kPpTokStride = 4 * kPpXWarps;        // a thread's tokens: tg + 32 i
constexpr int kPpTokPerThread = kPpM / kPpTokStride;  // 4
constexpr int kPpThreads = 64 + 32 * kPpXWarps;    // 320
constexpr int kPpTmemCols = 256;                   // two accumulators of 128 columns
constexpr int kPpCoef = kPpM * 20 * 4;           // a tile's post / comb, 10 KB
constexpr int kPpSmem = 1024 + kPpStages * (kPpAStage + kPpBStage) + kPpCoef + kPpM * 4 + 256;
constexpr int64_t kPpSms = 148;
constexpr int kPpMaxSplits = 16;

// Work plan: a tile's HB column blocks are cut into C chunks of L blocks (C <= 16); a chunk is one
// split of the partials (its rank in the tile), accumulated in one TMEM accumulator over at most
// 4 x 64 x L products per logit (fp32 accumulation error stays that of a short sum). The
// U = tiles x C chunks are dealt to P CTAs as equal contiguous ranges.
struct PpPlan {
  int64_t tiles, HB, L, C, U, P, S;  // S: splits of the partials (C rounded up to a power of two)
  size_t bw_bytes;
};

static PpPlan pp_plan(int64_t T, int64_t H) {
  PpPlan p;
  p.tiles = (T + kPpM - 1) / kPpM;
  p.HB = (H + kPpHB - 1) / kPpHB;
  p.L = (p.HB + kPpMaxSplits - 1) / kPpMaxSplits;
  p.C = (p.HB + p.L - 1) / p.L;
  p.U = p.tiles * p.C;
  p.P = p.U < kPpSms ? p.U : kPpSms;
  p.S = 1;
  while (p.S < p.C) p.S <<= 1;
  p.bw_bytes = (static_cast<size_t>(80) * 4 * H * 2 + 1023) / 1024 * 1024;
  return p;
}

bool post_project_supported(int64_t T, int64_t H) {
  return T >= 1 && H >= 8 && H % 8 == 0 && (T + kPpM - 1) / kPpM <= 0x7fffffff &&
         pp_plan(T, H).S <= kPpMaxSplits;
}

int post_project_splits(int64_t T, int64_t H) {
  return post_project_supported(T, H) ? static_cast<int>(pp_plan(T, H).S) : 0;
}

size_t post_project_workspace_bytes(int64_t T, int64_t H) {
  return post_project_supported(T, H) ? pp_plan(T, H).bw_bytes : 0;
}

// Logit j from the accumulator columns of its hi, mid and lo terms: (lo + mid) + hi.
__device__ __forceinline__ float pp_raw(const uint32_t (&d)[5][16], int j) {
  const float h3 = __uint_as_float(d[j / 16][j % 16]);
  const float m3 = __uint_as_float(d[(kMix + j) / 16][(kMix + j) % 16]);
  const float l3 = __uint_as_float(d[(2 * kMix + j) / 16][(2 * kMix + j) % 16]);
  return (l3 + m3) + h3;
}

__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gmem_src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)),
               "l"(gmem_src)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_prior() {  // all groups but the newest
  asm volatile("cp.async.wait_group 1;" ::: "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;" ::: "memory");
}

// Issues one block's residual copies for this thread's chunk ch (8 columns) of tokens
// tg + 32 i, i < 4, in all four streams, into stage s of the A tiles at their swizzled positions
// (zeros where the token or the column is out of range), as one commit group; and loads the
// block's x chunks into xn. The 8 lanes of a token cover one 128-byte row segment.
__device__ __forceinline__ void pp_issue_block(int64_t g, int64_t hb, int s, uint8_t* Abuf,
                                               const uint16_t* R, const uint16_t* x, int64_t T,
                                               int64_t H, int C, int tg, int ch,
                                               uint4 (&xn)[kPpTokPerThread]) {
  const int64_t t0 = (g / C) * kPpM;
  const int64_t h = hb * kPpHB + ch * 8;
#pragma unroll
  for (int i = 0; i < kPpTokPerThread; ++i) {
    const int r = tg + kPpTokStride * i;
    const int64_t t = t0 + r;
    uint8_t* dst = Abuf + s * kPpAStage + r * 128 + ((ch ^ (r & 7)) << 4);
    if (t < T && h < H) {
#pragma unroll
      for (int m = 0; m < 4; ++m) cp_async16(dst + m * kPpABytes, R + (t * 4 + m) * H + h);
      xn[i] = __ldg(reinterpret_cast<const uint4*>(x + t * H + h));
    } else {
#pragma unroll
      for (int m = 0; m < 4; ++m)
        *reinterpret_cast<uint4*>(dst + m * kPpABytes) = make_uint4(0u, 0u, 0u, 0u);
      xn[i] = make_uint4(0u, 0u, 0u, 0u);
    }
  }
  cp_async_commit();
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

__global__ void __launch_bounds__(kPpThreads, 1) post_project_kernel(
    const __grid_constant__ CUtensorMap tmB, const uint16_t* __restrict__ x, const uint16_t* R,
    const float* __restrict__ post, const float* __restrict__ comb, uint16_t* out,
    float* __restrict__ dot_mix, float* __restrict__ sqrsum, int64_t T, int64_t H, int64_t U,
    int HB, int L, int C, int S) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_u32 = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + (((raw_u32 + 1023u) & ~1023u) - raw_u32);
  uint8_t* Abuf = smem;                                   // [2][4][128 x 128 B]
  uint8_t* Bbuf = smem + kPpStages * kPpAStage;           // [2][4][80 x 128 B]
  float* coef_s = reinterpret_cast<float*>(Bbuf + kPpStages * kPpBStage);  // [128][20]
  float* ss_s = coef_s + kPpM * 20;                                            // [128]
  uint64_t* bars = reinterpret_cast<uint64_t*>(ss_s + kPpM);
  uint64_t* afull = bars;        // [2] 8 post-map warps wrote the A tiles
  uint64_t* aempty = bars + 2;   // [2] MMAs done with them
  uint64_t* bfull = bars + 4;    // [2] TMA bytes
  uint64_t* bempty = bars + 6;   // [2]
  uint64_t* accfull = bars + 8;  // [2]
  uint64_t* accempty = bars + 10;  // [2] 8 post-map warps read the accumulator
  uint64_t* done = bars + 12;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 13);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int64_t P = gridDim.x;
  const int64_t c = blockIdx.x;
  const int64_t lo = c * U / P, hi = (c + 1) * U / P;  // chunks of this CTA

  if (threadIdx.x == 0) {
    for (int s = 0; s < kPpStages; ++s) {
      mbar_init(&afull[s], kPpXWarps);
      mbar_init(&aempty[s], 1);
      mbar_init(&bfull[s], 1);
      mbar_init(&bempty[s], 1);
      mbar_init(&accfull[s], 1);
      mbar_init(&accempty[s], kPpEpiWarps);
    }
    mbar_init(done, 1);
    fence_mbarrier_init();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(tmem_slot)),
                 "r"(kPpTmemCols)
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
      int64_t n = 0;
      bool ok = true;
      for (int64_t g = lo; g < hi && ok; ++g) {
        const int64_t hbs = (g % C) * L;
        const int64_t hbe = min(static_cast<int64_t>(HB), hbs + L);
        for (int64_t hb = hbs; hb < hbe; ++hb, ++n) {
          const int s = static_cast<int>(n & 1);
          if (n >= kPpStages &&
              !mbar_wait(&bempty[s], static_cast<uint32_t>((n >> 1) - 1) & 1u, 40)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&bfull[s], kPpBStage);
#pragma unroll
          for (int st = 0; st < 4; ++st)
            tma_load_2d(Bbuf + s * kPpBStage + st * kPpBBytes, &tmB,
                        static_cast<int>(st * H + hb * kPpHB), 0, &bfull[s]);
        }
      }
      if (!ok) {
        for (int64_t i = n - kPpStages; i < n; ++i)
          if (i >= 0) mbar_wait(&bfull[i & 1], static_cast<uint32_t>(i >> 1) & 1u, 41);
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      int64_t n = 0, p = 0;
      bool ok = true;
      for (int64_t g = lo; g < hi && ok; ++g, ++p) {
        const int64_t hbs = (g % C) * L;
        const int64_t hbe = min(static_cast<int64_t>(HB), hbs + L);
        const int b = static_cast<int>(p & 1);
        if (p >= 2 && !mbar_wait(&accempty[b], static_cast<uint32_t>((p >> 1) - 1) & 1u, 42)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t dt = tmem + static_cast<uint32_t>(b * 128);
        for (int64_t hb = hbs; hb < hbe; ++hb, ++n) {
          const int s = static_cast<int>(n & 1);
          const uint32_t ph = static_cast<uint32_t>(n >> 1) & 1u;
          if (!mbar_wait(&afull[s], ph, 43) || !mbar_wait(&bfull[s], ph, 44)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_u32(Abuf + s * kPpAStage);
          const uint32_t b0 = smem_u32(Bbuf + s * kPpBStage);
#pragma unroll
          for (int st = 0; st < 4; ++st) {
            const uint64_t adesc = sw128_desc(a0 + st * kPpABytes);
            const uint64_t bdesc = sw128_desc(b0 + st * kPpBBytes);
#pragma unroll
            for (int k = 0; k < kPpHB / 16; ++k)
              umma_bf16(dt, adesc + 2 * k, bdesc + 2 * k,
                        (hb > hbs || st > 0 || k > 0) ? 1u : 0u);
          }
          umma_commit(&aempty[s]);
          umma_commit(&bempty[s]);
        }
        if (!ok) break;
        umma_commit(&accfull[b]);
      }
      umma_commit(done);
      mbar_wait(done, 0, 45);
    }
  } else {
    // ------------------------------------------------------------------ post-map warps
    const int xt = threadIdx.x - 64;  // 0..255
    const int ch = xt & 7;            // 8-column chunk of the block
    const int tg = xt >> 3;           // tokens tg + 32 i, i < 4
    const int xw = warp - 2;          // 0..7
    int64_t n = 0, p = 0;
    bool dead = false;
    // Block n's residual arrives in stage n & 1 by 16-byte asynchronous copies issued one block
    // ahead (each thread copies, and later reads, only its own rows and chunk); its x chunks are
    // loaded into registers one block ahead too. The post-map then overwrites the stage in place
    // with out, which is the MMA's A operand.
    uint4 xnext[kPpTokPerThread];
    if (lo < hi) pp_issue_block(lo, (lo % C) * L, 0, Abuf, R, x, T, H, C, tg, ch, xnext);
    for (int64_t g = lo; g < hi; ++g, ++p) {
      const int64_t tile = g / C;
      const int64_t slot = g - tile * C;  // the chunk's rank in its tile: its split
      const int64_t hbs = slot * L;
      const int64_t hbe = min(static_cast<int64_t>(HB), hbs + L);
      // The tile's post / comb into shared memory (the previous chunk's readers are past the
      // epilogue's barriers): 128 tokens x 5 float4.
      for (int e = xt; e < kPpM * 5; e += 32 * kPpXWarps) {
        const int r = e / 5, v = e - r * 5;
        const int64_t t = tile * kPpM + r;
        float4 val = make_float4(0.f, 0.f, 0.f, 0.f);
        if (t < T)
          val = v == 0 ? __ldg(reinterpret_cast<const float4*>(post + t * 4))
                       : __ldg(reinterpret_cast<const float4*>(comb + t * 16 + (v - 1) * 4));
        reinterpret_cast<float4*>(coef_s)[r * 5 + v] = val;
      }
      dead = named_bar_or(1, 32 * kPpXWarps, dead);
      float ss[kPpTokPerThread];
#pragma unroll
      for (int i = 0; i < kPpTokPerThread; ++i) ss[i] = 0.f;
      for (int64_t hb = hbs; hb < hbe; ++hb, ++n) {
        const int s = static_cast<int>(n & 1);
        uint4 xv[kPpTokPerThread];
#pragma unroll
        for (int i = 0; i < kPpTokPerThread; ++i) xv[i] = xnext[i];
        // Next block: into stage s ^ 1, once the MMAs of block n - 1 (its last user) are done.
        const bool more = hb + 1 < hbe || g + 1 < hi;
        if (more && n >= 1 && !dead)
          dead = !__all_sync(0xffffffffu, mbar_wait(&aempty[s ^ 1],
                                                   static_cast<uint32_t>((n - 1) >> 1) & 1u, 46));
        if (more && !dead) {
          if (hb + 1 < hbe)
            pp_issue_block(g, hb + 1, s ^ 1, Abuf, R, x, T, H, C, tg, ch, xnext);
          else
            pp_issue_block(g + 1, ((g + 1) % C) * L, s ^ 1, Abuf, R, x, T, H, C, tg, ch, xnext);
        } else {
          cp_async_commit();  // an empty group keeps the group count per block
        }
        cp_async_wait_prior();  // this block's copies (all groups but the newest) have landed
        if (dead) continue;
        const int64_t h = hb * kPpHB + ch * 8;
#pragma unroll
        for (int i = 0; i < kPpTokPerThread; ++i) {
          const int r = tg + kPpTokStride * i;
          const int64_t t = tile * kPpM + r;
          const bool valid = t < T && h < H;
          uint8_t* As = Abuf + s * kPpAStage + r * 128 + ((ch ^ (r & 7)) << 4);
          const float4* cs = reinterpret_cast<const float4*>(coef_s) + r * 5;
          Coef20 k20;
          k20.post = cs[0];
#pragma unroll
          for (int o = 0; o < 4; ++o) k20.c[o] = cs[1 + o];
          uint4 rv[4], ov[4];
#pragma unroll
          for (int m = 0; m < 4; ++m) rv[m] = *reinterpret_cast<const uint4*>(As + m * kPpABytes);
          mix_vec8(xv[i], rv, k20, ov);
          if (!valid) {
#pragma unroll
            for (int m = 0; m < 4; ++m) ov[m] = make_uint4(0u, 0u, 0u, 0u);
          }
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            if (valid) __stcg(reinterpret_cast<uint4*>(out + (t * 4 + m) * H + h), ov[m]);
            *reinterpret_cast<uint4*>(As + m * kPpABytes) = ov[m];
            const uint32_t w4[4] = {ov[m].x, ov[m].y, ov[m].z, ov[m].w};
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const float a = bf16_lo(w4[q]), b = bf16_hi(w4[q]);
              ss[i] = fmaf(a, a, ss[i]);
              ss[i] = fmaf(b, b, ss[i]);
            }
          }
        }
        fence_proxy_async_smem();  // generic-proxy writes -> the MMA's async-proxy reads
        __syncwarp();
        if (lane == 0) mbar_arrive(&afull[s]);
      }
      // ---------------------------------------------------------------- piece epilogue
      // A token's 8 chunk lanes are consecutive lanes: a fixed xor tree joins them.
#pragma unroll
      for (int i = 0; i < kPpTokPerThread; ++i) {
        float v = ss[i];
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        if (ch == 0) ss_s[tg + kPpTokStride * i] = v;
      }
      dead = named_bar_or(1, 32 * kPpXWarps, dead);
      const int b = static_cast<int>(p & 1);
      const bool epi = xw < kPpEpiWarps;  // warps 2..9 read the accumulator
      if (epi && !dead)
        dead = !__all_sync(0xffffffffu,
                           mbar_wait(&accfull[b], static_cast<uint32_t>(p >> 1) & 1u, 47));
      if (epi && !dead) {
        tc_fence_after();
        const int q = warp & 3;  // a warp reads TMEM lanes 32 * (warp % 4) .. + 31
        const int jh = xw >> 2;  // logits 12*jh .. 12*jh+11 (warps 2-5: 0, warps 6-9: 1)
        const int row = q * 32 + lane;
        const uint32_t tb =
            tmem + static_cast<uint32_t>(b * 128) + (static_cast<uint32_t>(q * 32) << 16);
        uint32_t d[5][16];  // columns 0..79: hi 0..23 | mid 24..47 | lo 48..71 | zero rows
#pragma unroll
        for (int cc = 0; cc < 5; ++cc) tmem_ld16(tb + cc * 16, d[cc]);
        tmem_wait_ld();
        const int64_t tr = tile * kPpM + row;
        if (tr < T) {
          float raw[12];
          if (jh == 0) {
#pragma unroll
            for (int j = 0; j < 12; ++j) raw[j] = pp_raw(d, j);
          } else {
#pragma unroll
            for (int j = 0; j < 12; ++j) raw[j] = pp_raw(d, 12 + j);
          }
          float4* dst = reinterpret_cast<float4*>(dot_mix + (slot * T + tr) * kMix + jh * 12);
#pragma unroll
          for (int v = 0; v < 3; ++v)
            dst[v] = make_float4(raw[4 * v], raw[4 * v + 1], raw[4 * v + 2], raw[4 * v + 3]);
          if (jh == 0) sqrsum[slot * T + tr] = ss_s[row];
          if (slot == C - 1) {  // the tile's last chunk: zero the splits beyond C
            const float4 z = make_float4(0.f, 0.f, 0.f, 0.f);
            for (int64_t sl = slot + 1; sl < S; ++sl) {
              float4* zr = reinterpret_cast<float4*>(dot_mix + (sl * T + tr) * kMix + jh * 12);
#pragma unroll
              for (int v = 0; v < 3; ++v) zr[v] = z;
              if (jh == 0) sqrsum[sl * T + tr] = 0.f;
            }
          }
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&accempty[b]);
      }
      // ss_s is rewritten at the next piece's end only after every warp has read it here.
      dead = named_bar_or(1, 32 * kPpXWarps, dead);
    }
  }
  cp_async_wait_all();  // no copy into shared memory outlives the CTA
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                 "r"(kPpTmemCols)
                 : "memory");
  }
}

int launch_post_project(const PostProjectArgs& a, cudaStream_t s) {
  const PpPlan plan = pp_plan(a.T, a.H);
  const int64_t K = 4 * a.H;
  uint16_t* Bw = static_cast<uint16_t*>(a.workspace);
  CUtensorMap mB;
  if (!make_map(&mB, Bw, K, 80, 80)) return -4;
  if (!ensure_smem_limit(reinterpret_cast<const void*>(post_project_kernel), kPpSmem)) return -4;
  const int64_t sb = (K + 255) / 256;
  if (launch_pdl(pre_tc_split_kernel, dim3(static_cast<unsigned>(sb < 4096 ? sb : 4096)),
                 dim3(256), 0, s, a.hc_fn, Bw, K) != cudaSuccess)
    return -4;
  note_launches(1);
  if (launch_pdl(post_project_kernel, dim3(static_cast<unsigned>(plan.P)), dim3(kPpThreads),
                 static_cast<size_t>(kPpSmem), s, mB, a.x, a.R, a.post, a.comb, a.out, a.dot_mix,
                 a.sqrsum, a.T, a.H, plan.U, static_cast<int>(plan.HB), static_cast<int>(plan.L),
                 static_cast<int>(plan.C), static_cast<int>(plan.S)) != cudaSuccess)
    return -4;
  note_launches(1);
  return 0;
}

}  // namespace mhc
