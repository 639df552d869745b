// C ABI of libmhc.so (declared in include/mhc.h): host-side validation, alias checks, device
// binding and kernel dispatch. Nothing is launched before every check has passed
// (glm5next_mhc.rs glm_hc_pre: refuse before launching; "FlashInfer mHC module deep dive" §2.3:
// an empty input returns without a launch, §3.2: eps > 0 and sinkhorn_repeat >= 1).
#include <math.h>

#include <atomic>
#include <mutex>

#include "mhc.h"
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

namespace {
constexpr int kMaxDevices = 64;
int g_sm_count[kMaxDevices] = {};
int g_cc[kMaxDevices] = {};
std::mutex g_mu;

void query_device(int dev) {
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_sm_count[dev] != 0) return;
  int sms = 0, major = 0, minor = 0;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
  cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev);
  g_cc[dev] = major * 10 + minor;
  g_sm_count[dev] = sms > 0 ? sms : 1;
}
}  // namespace

namespace {
struct SmemLimit {
  const void* kernel;
  int device;
  int bytes;
};
constexpr int kMaxSmemLimits = 256;
SmemLimit g_smem_limits[kMaxSmemLimits];
int g_n_smem_limits = 0;
std::mutex g_smem_mu;
}  // namespace

bool ensure_smem_limit(const void* kernel, int bytes) {
  const int dev = current_device();
  if (dev < 0) return false;
  std::lock_guard<std::mutex> lock(g_smem_mu);
  for (int i = 0; i < g_n_smem_limits; ++i)
    if (g_smem_limits[i].kernel == kernel && g_smem_limits[i].device == dev &&
        g_smem_limits[i].bytes >= bytes)
      return true;
  if (cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) !=
      cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  if (g_n_smem_limits < kMaxSmemLimits) g_smem_limits[g_n_smem_limits++] = {kernel, dev, bytes};
  return true;
}

static std::atomic<uint64_t> g_launches{0};

// Health check of the bounded waits: one thread waits on an mbarrier that nothing arrives at, with
// the caller's limit instead of the library-wide one, through the same wait routine the pipelines
// use. No copy or MMA is in flight, so giving up leaves nothing behind.
__global__ void selftest_wait_kernel(unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    fence_mbarrier_init();
    mbar_wait_for(&bar, 0, 99, limit_ns);
  }
}
void note_launches(int n) { g_launches.fetch_add(static_cast<uint64_t>(n), std::memory_order_relaxed); }

int current_device() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return -1;
  return dev;
}

int device_sm_count() {
  const int dev = current_device();
  if (dev < 0) return 1;
  if (g_sm_count[dev] == 0) query_device(dev);
  return g_sm_count[dev];
}

int device_cc() {
  const int dev = current_device();
  if (dev < 0) return 0;
  if (g_sm_count[dev] == 0) query_device(dev);
  return g_cc[dev];
}

// Make this runtime's current device the one that owns `p` (the caller's framework may have a
// different device current), and check that `p` is device memory and the device is sm_100.
static int bind_device(const void* p) {
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, p) != cudaSuccess) {
    cudaGetLastError();
    return MHC_ERR_INVALID_ARG;
  }
  if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return MHC_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return MHC_ERR_CUDA;
  if (cur != at.device && cudaSetDevice(at.device) != cudaSuccess) return MHC_ERR_CUDA;
  if (device_cc() / 10 != 10) return MHC_ERR_UNSUPPORTED;
  return MHC_OK;
}

// Byte ranges [a, a+na) and [b, b+nb) intersect.
static bool overlaps(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na > 0 && nb > 0 && x < y + nb && y < x + na;
}

constexpr int64_t kPreTensorMinTokens = 128;
constexpr int64_t kPostPersistentMinH = 2048;
constexpr int64_t kPostPersistentMinElems = int64_t(1) << 22;

static bool mul_ok(int64_t a, int64_t b, int64_t limit) { return a >= 0 && b >= 0 && (b == 0 || a <= limit / b); }

}  // namespace mhc

using namespace mhc;

extern "C" {

mhc_params mhc_default_params(void) {
  mhc_params p;
  p.sinkhorn_iters = 20;
  p.sinkhorn_eps = 1e-6f;
  p.rms_eps = 1e-6f;
  p.pre_eps = 0.0f;
  p.post_mult = 2.0f;
  return p;
}

const char* mhc_status_string(int status) {
  switch (status) {
    case MHC_OK: return "MHC_OK";
    case MHC_ERR_INVALID_ARG: return "MHC_ERR_INVALID_ARG";
    case MHC_ERR_WORKSPACE_TOO_SMALL: return "MHC_ERR_WORKSPACE_TOO_SMALL";
    case MHC_ERR_ALIAS: return "MHC_ERR_ALIAS";
    case MHC_ERR_CUDA: return "MHC_ERR_CUDA";
    case MHC_ERR_UNSUPPORTED: return "MHC_ERR_UNSUPPORTED";
    case MHC_ERR_TIMEOUT: return "MHC_ERR_TIMEOUT";
    case MHC_ERR_SCRATCH_LIMIT: return "MHC_ERR_SCRATCH_LIMIT";
    default: return "MHC_ERR_UNKNOWN";
  }
}

int mhc_version(void) { return 100; }

uint64_t mhc_launch_count(void) { return g_launches.load(std::memory_order_relaxed); }

size_t mhc_pre_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0) return 0;
  size_t m = pre_cc_workspace_bytes(T, H);
  const size_t b = pre_tc_workspace_bytes(T, H), c = pre_fused_workspace_bytes(T, H);
  const size_t d = pre_wave_workspace_bytes(T, H);
  if (b > m) m = b;
  if (c > m) m = c;
  if (d > m) m = d;
  return (m + 255) / 256 * 256;
}

int mhc_post_with_path(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                       uint16_t* out, int64_t T, int64_t H, int path, mhc_stream_t stream) {
  if (T < 0 || H <= 0) return MHC_ERR_INVALID_ARG;
  if (!mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!x || !R || !post || !comb || !out) return MHC_ERR_INVALID_ARG;
  const size_t nR = static_cast<size_t>(T) * 4 * H * 2, nx = static_cast<size_t>(T) * H * 2;
  if (static_cast<const void*>(out) != static_cast<const void*>(R) && overlaps(out, nR, R, nR))
    return MHC_ERR_ALIAS;
  if (overlaps(out, nR, x, nx) || overlaps(out, nR, post, T * 16) || overlaps(out, nR, comb, T * 64))
    return MHC_ERR_ALIAS;
  const bool vec_ok = (H % 8 == 0) && aligned16(x) && aligned16(R) && aligned16(out) &&
                      aligned16(post) && aligned16(comb);
  if (path == MHC_PATH_AUTO) {
    // The bulk-copy staged persistent kernel streams best once rows are long (one 1024-element
    // chunk per tile row) and the call is large; short rows and small calls take vec8.
    const bool big = H >= kPostPersistentMinH && T * H >= kPostPersistentMinElems;
    path = !vec_ok ? MHC_POST_PATH_SCALAR : (big ? MHC_POST_PATH_PERSISTENT : MHC_POST_PATH_VEC8);
  } else if (path == MHC_POST_PATH_VEC8 || path == MHC_POST_PATH_PERSISTENT) {
    if (!vec_ok) return MHC_ERR_UNSUPPORTED;
  } else if (path != MHC_POST_PATH_SCALAR) {
    return MHC_ERR_INVALID_ARG;
  }
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (path == MHC_POST_PATH_VEC8) return launch_post_vec8(x, R, post, comb, out, T, H, s);
  if (path == MHC_POST_PATH_PERSISTENT) return launch_post_persistent(x, R, post, comb, out, T, H, s);
  return launch_post_scalar(x, R, post, comb, out, T, H, s);
}

int mhc_post(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
             uint16_t* out, int64_t T, int64_t H, mhc_stream_t stream) {
  return mhc_post_with_path(x, R, post, comb, out, T, H, MHC_PATH_AUTO, stream);
}

int mhc_sinkhorn(const float* logits, float* comb, int64_t T, int64_t H_unused, int iters,
                 float eps, mhc_stream_t stream) {
  (void)H_unused;
  if (T < 0 || iters < 1 || !(eps > 0.0f) || !isfinite(eps)) return MHC_ERR_INVALID_ARG;
  if (!mul_ok(T, 64, INT64_MAX)) return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!logits || !comb) return MHC_ERR_INVALID_ARG;
  const size_t n = static_cast<size_t>(T) * 64;
  if (static_cast<const void*>(comb) != static_cast<const void*>(logits) && overlaps(comb, n, logits, n))
    return MHC_ERR_ALIAS;
  int st = bind_device(logits);
  if (st != MHC_OK) return st;
  return launch_sinkhorn(logits, comb, T, iters, eps, reinterpret_cast<cudaStream_t>(stream));
}

int mhc_pre_with_path(const uint16_t* R, const float* hc_fn, const float* hc_scale,
                      const float* hc_base, uint16_t* y, float* pre, float* post, float* comb,
                      void* workspace, size_t workspace_bytes, int64_t T, int64_t H,
                      const mhc_params* p, int path, mhc_stream_t stream) {
  const mhc_params prm = p ? *p : mhc_default_params();
  if (T < 0 || H <= 0) return MHC_ERR_INVALID_ARG;
  if (!mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (prm.sinkhorn_iters < 1 || !(prm.sinkhorn_eps > 0.0f) || !isfinite(prm.sinkhorn_eps) ||
      !(prm.rms_eps > 0.0f) || !isfinite(prm.rms_eps) || !(prm.pre_eps >= 0.0f) ||
      !isfinite(prm.pre_eps) || !isfinite(prm.post_mult))
    return MHC_ERR_INVALID_ARG;
  if (path != MHC_PATH_AUTO && path != MHC_PRE_PATH_CUDA_CORE && path != MHC_PRE_PATH_TENSOR &&
      path != MHC_PRE_PATH_TENSOR_SPLIT && path != MHC_PRE_PATH_TENSOR_FUSED &&
      path != MHC_PRE_PATH_TENSOR_WAVE)
    return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!R || !hc_fn || !hc_scale || !hc_base || !y || !pre || !post || !comb)
    return MHC_ERR_INVALID_ARG;
  const size_t need = mhc_pre_workspace_bytes(T, H);
  if (workspace_bytes < need || (need > 0 && workspace == nullptr)) return MHC_ERR_WORKSPACE_TOO_SMALL;
  const size_t nR = static_cast<size_t>(T) * 4 * H * 2, ny = static_cast<size_t>(T) * H * 2;
  const size_t n4 = static_cast<size_t>(T) * 16, n16 = static_cast<size_t>(T) * 64;
  const void* outs[4] = {y, pre, post, comb};
  const size_t outn[4] = {ny, n4, n4, n16};
  const void* ins[5] = {R, hc_fn, hc_scale, hc_base, workspace};
  const size_t inn[5] = {nR, static_cast<size_t>(H) * 4 * 24 * 4, 12, 96, need};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 5; ++j)
      if (ins[j] && overlaps(outs[i], outn[i], ins[j], inn[j])) return MHC_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], outn[i], outs[j], outn[j])) return MHC_ERR_ALIAS;
  }
  if (workspace && (overlaps(workspace, need, R, nR) || overlaps(workspace, need, hc_fn, inn[1])))
    return MHC_ERR_ALIAS;
  // The tensor path reads R and its split hc_fn copy (in the workspace) with TMA: 16-byte aligned
  // bases. Below kPreTensorMinTokens the CUDA-core path, which reads hc_fn once in fp32, is faster.
  const bool tc_ok = pre_tc_supported(T, H) && aligned16(R) && aligned16(workspace);
  // The fused kernel also uses 16-byte accesses on y, pre and comb.
  const bool fused_ok = tc_ok && pre_fused_supported(T, H) && aligned16(y) && aligned16(pre) &&
                        aligned16(comb);
  // The wavefront single pass: 16-byte accesses on y and comb as well.
  const bool wave_ok =
      tc_ok && pre_wave_supported(T, H) && aligned16(y) && aligned16(comb);
  bool auto_fused = false;
  if (path == MHC_PATH_AUTO) {
    path = (tc_ok && T >= kPreTensorMinTokens) ? MHC_PRE_PATH_TENSOR : MHC_PRE_PATH_CUDA_CORE;
    auto_fused = path == MHC_PRE_PATH_TENSOR && fused_ok && pre_fused_preferred(T, H);
  } else if ((path == MHC_PRE_PATH_TENSOR || path == MHC_PRE_PATH_TENSOR_SPLIT) && !tc_ok) {
    return MHC_ERR_UNSUPPORTED;
  } else if (path == MHC_PRE_PATH_TENSOR_FUSED && !fused_ok) {
    return MHC_ERR_UNSUPPORTED;
  } else if (path == MHC_PRE_PATH_TENSOR_WAVE && !wave_ok) {
    return MHC_ERR_UNSUPPORTED;
  }
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  PreArgs a{R, hc_fn, hc_scale, hc_base, y, pre, post, comb, workspace, workspace_bytes, T, H,
            prm.sinkhorn_iters, prm.sinkhorn_eps, prm.rms_eps, prm.pre_eps, prm.post_mult};
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (path == MHC_PRE_PATH_TENSOR_WAVE) {
    // 1: the grid cannot run with every CTA resident on this device; nothing was launched.
    const int r = launch_pre_wave(a, s);
    return r == 1 ? MHC_ERR_UNSUPPORTED : r;
  }
  if (path == MHC_PRE_PATH_TENSOR_FUSED || auto_fused) {
    // 1: the grid cannot run with every CTA resident on this device; nothing was launched. A
    // forced single pass reports it; the automatic choice falls back to the split chain.
    const int r = launch_pre_fused(a, s);
    if (r != 1) return r;
    if (!auto_fused) return MHC_ERR_UNSUPPORTED;
  }
  if (path != MHC_PRE_PATH_CUDA_CORE) return launch_pre_tc(a, s);
  return launch_pre_cc(a, s);
}

int mhc_pre(const uint16_t* R, const float* hc_fn, const float* hc_scale, const float* hc_base,
            uint16_t* y, float* pre, float* post, float* comb, void* workspace,
            size_t workspace_bytes, int64_t T, int64_t H, const mhc_params* p,
            mhc_stream_t stream) {
  return mhc_pre_with_path(R, hc_fn, hc_scale, hc_base, y, pre, post, comb, workspace,
                           workspace_bytes, T, H, p, MHC_PATH_AUTO, stream);
}

static int pre_big_fuse_common(const float* dot_mix, const float* sqrsum, int num_splits,
                               double k, const uint16_t* R, const float* hc_scale,
                               const float* hc_base, uint16_t* y, float* pre, float* post,
                               float* comb, int64_t T, int64_t H, const mhc_params* p,
                               mhc_stream_t stream) {
  const mhc_params prm = p ? *p : mhc_default_params();
  if (T < 0 || H <= 0) return MHC_ERR_INVALID_ARG;
  if (!mul_ok(T, 4 * H, INT64_MAX / 4) || !mul_ok(T, 96 * num_splits, INT64_MAX)) return MHC_ERR_INVALID_ARG;
  if (num_splits != 1 && num_splits != 2 && num_splits != 4 && num_splits != 8 && num_splits != 16)
    return MHC_ERR_INVALID_ARG;
  if (!(k > 0.0) || !(k < 3.0e38)) return MHC_ERR_INVALID_ARG;
  if (prm.sinkhorn_iters < 1 || !(prm.sinkhorn_eps > 0.0f) || !isfinite(prm.sinkhorn_eps) ||
      !(prm.rms_eps > 0.0f) || !isfinite(prm.rms_eps) || !(prm.pre_eps >= 0.0f) ||
      !isfinite(prm.pre_eps) || !isfinite(prm.post_mult))
    return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!dot_mix || !R || !hc_scale || !hc_base || !y || !pre || !post || !comb)
    return MHC_ERR_INVALID_ARG;
  const size_t nR = static_cast<size_t>(T) * 4 * H * 2, ny = static_cast<size_t>(T) * H * 2;
  const size_t n4 = static_cast<size_t>(T) * 16, n16 = static_cast<size_t>(T) * 64;
  const size_t nd = static_cast<size_t>(T) * 96 * num_splits, ns = static_cast<size_t>(T) * 4 * num_splits;
  const void* outs[4] = {y, pre, post, comb};
  const size_t outn[4] = {ny, n4, n4, n16};
  const void* ins[5] = {dot_mix, sqrsum, R, hc_scale, hc_base};
  const size_t inn[5] = {nd, ns, nR, 12, 96};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 5; ++j)
      if (ins[j] && overlaps(outs[i], outn[i], ins[j], inn[j])) return MHC_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], outn[i], outs[j], outn[j])) return MHC_ERR_ALIAS;
  }
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  BigFuseArgs a{dot_mix, sqrsum, num_splits, static_cast<float>(k), R, hc_scale, hc_base, y, pre,
                post, comb, T, H, prm.sinkhorn_iters, prm.sinkhorn_eps, prm.rms_eps, prm.pre_eps,
                prm.post_mult};
  return launch_pre_bigfuse(a, reinterpret_cast<cudaStream_t>(stream));
}

int mhc_pre_big_fuse(const float* dot_mix, const float* sqrsum, int num_splits, int64_t k,
                     const uint16_t* R, const float* hc_scale, const float* hc_base, uint16_t* y,
                     float* pre, float* post, float* comb, int64_t T, int64_t H,
                     const mhc_params* p, mhc_stream_t stream) {
  if (!sqrsum && T > 0) return MHC_ERR_INVALID_ARG;
  if (k < 1) return MHC_ERR_INVALID_ARG;
  return pre_big_fuse_common(dot_mix, sqrsum, num_splits, static_cast<double>(k), R, hc_scale,
                             hc_base, y, pre, post, comb, T, H, p, stream);
}

int mhc_pre_big_fuse_with_prenorm(const float* dot_mix, const uint16_t* R, const float* hc_scale,
                                  const float* hc_base, uint16_t* y, float* pre, float* post,
                                  float* comb, int64_t T, int64_t H, const mhc_params* p,
                                  mhc_stream_t stream) {
  return pre_big_fuse_common(dot_mix, nullptr, 1, 4.0 * static_cast<double>(H), R, hc_scale,
                             hc_base, y, pre, post, comb, T, H, p, stream);
}

int mhc_post_project_splits(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return 0;
  return post_project_splits(T, H);
}

size_t mhc_post_project_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return 0;
  const size_t b = post_project_workspace_bytes(T, H);
  return (b + 255) / 256 * 256;
}

int mhc_post_project(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                     uint16_t* out, const float* hc_fn_next, float* dot_mix, float* sqrsum,
                     void* workspace, size_t workspace_bytes, int64_t T, int64_t H,
                     mhc_stream_t stream) {
  if (T < 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!x || !R || !post || !comb || !out || !hc_fn_next || !dot_mix || !sqrsum)
    return MHC_ERR_INVALID_ARG;
  if (!post_project_supported(T, H) || !aligned16(x) || !aligned16(R) || !aligned16(out) ||
      !aligned16(post) || !aligned16(comb) || !aligned16(dot_mix))
    return MHC_ERR_UNSUPPORTED;
  const size_t need = mhc_post_project_workspace_bytes(T, H);
  if (workspace_bytes < need || !workspace) return MHC_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MHC_ERR_INVALID_ARG;
  const int S = post_project_splits(T, H);
  const size_t nR = static_cast<size_t>(T) * 8 * H, nx = static_cast<size_t>(T) * H * 2;
  const size_t nd = static_cast<size_t>(S) * T * 96, ns = static_cast<size_t>(S) * T * 4;
  const size_t nfn = static_cast<size_t>(4 * H) * 96;
  if (static_cast<const void*>(out) != static_cast<const void*>(R) && overlaps(out, nR, R, nR))
    return MHC_ERR_ALIAS;
  const void* outs[4] = {out, dot_mix, sqrsum, workspace};
  const size_t outn[4] = {nR, nd, ns, need};
  const void* ins[5] = {x, post, comb, hc_fn_next, R};
  const size_t inn[5] = {nx, static_cast<size_t>(T) * 16, static_cast<size_t>(T) * 64, nfn, nR};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 5; ++j) {
      if (i == 0 && j == 4) continue;  // out == R is allowed (checked above)
      if (overlaps(outs[i], outn[i], ins[j], inn[j])) return MHC_ERR_ALIAS;
    }
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], outn[i], outs[j], outn[j])) return MHC_ERR_ALIAS;
  }
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  PostProjectArgs a{x, R, post, comb, out, hc_fn_next, dot_mix, sqrsum, workspace, T, H};
  return launch_post_project(a, reinterpret_cast<cudaStream_t>(stream));
}

int mhc_post_backward(const uint16_t* d_out, const uint16_t* x, const uint16_t* R,
                      const float* post, const float* comb, uint16_t* d_x, uint16_t* d_R,
                      float* d_post, float* d_comb, int64_t T, int64_t H, mhc_stream_t stream) {
  if (T < 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!d_out || !x || !R || !post || !comb || !d_x || !d_R || !d_post || !d_comb)
    return MHC_ERR_INVALID_ARG;
  const size_t nR = static_cast<size_t>(T) * 8 * H, nx = static_cast<size_t>(T) * H * 2;
  const void* outs[4] = {d_x, d_R, d_post, d_comb};
  const size_t outn[4] = {nx, nR, static_cast<size_t>(T) * 16, static_cast<size_t>(T) * 64};
  const void* ins[5] = {d_out, x, R, post, comb};
  const size_t inn[5] = {nR, nx, nR, static_cast<size_t>(T) * 16, static_cast<size_t>(T) * 64};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 5; ++j)
      if (overlaps(outs[i], outn[i], ins[j], inn[j])) return MHC_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (overlaps(outs[i], outn[i], outs[j], outn[j])) return MHC_ERR_ALIAS;
  }
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  return launch_post_backward(d_out, x, R, post, comb, d_x, d_R, d_post, d_comb, T, H,
                              reinterpret_cast<cudaStream_t>(stream));
}

size_t mhc_pre_backward_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return 0;
  return pre_backward_workspace_bytes(T, H);
}

int mhc_pre_backward(const uint16_t* d_y, const float* d_pre, const float* d_post,
                     const float* d_comb, const uint16_t* R, const float* hc_fn,
                     const float* hc_scale, const float* hc_base, uint16_t* d_R, float* d_hc_fn,
                     float* d_scale, float* d_base, void* workspace, size_t workspace_bytes,
                     int64_t T, int64_t H, const mhc_params* p, mhc_stream_t stream) {
  const mhc_params prm = p ? *p : mhc_default_params();
  if (T < 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (prm.sinkhorn_iters < 1 || !(prm.sinkhorn_eps > 0.0f) || !isfinite(prm.sinkhorn_eps) ||
      !(prm.rms_eps > 0.0f) || !isfinite(prm.rms_eps) || !(prm.pre_eps >= 0.0f) ||
      !isfinite(prm.pre_eps) || !isfinite(prm.post_mult))
    return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!R || !hc_fn || !hc_scale || !hc_base || !d_R || !d_hc_fn || !d_scale || !d_base)
    return MHC_ERR_INVALID_ARG;
  const size_t need = mhc_pre_backward_workspace_bytes(T, H);
  if (workspace_bytes < need || !workspace) return MHC_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MHC_ERR_INVALID_ARG;
  const size_t nR = static_cast<size_t>(T) * 8 * H, ny = static_cast<size_t>(T) * H * 2;
  const size_t nfn = static_cast<size_t>(4 * H) * 96;
  const void* outs[5] = {d_R, d_hc_fn, d_scale, d_base, workspace};
  const size_t outn[5] = {nR, nfn, 12, 96, need};
  const void* ins[8] = {d_y, d_pre, d_post, d_comb, R, hc_fn, hc_scale, hc_base};
  const size_t inn[8] = {ny, static_cast<size_t>(T) * 16, static_cast<size_t>(T) * 16,
                         static_cast<size_t>(T) * 64, nR, nfn, 12, 96};
  for (int i = 0; i < 5; ++i) {
    for (int j = 0; j < 8; ++j)
      if (ins[j] && overlaps(outs[i], outn[i], ins[j], inn[j])) return MHC_ERR_ALIAS;
    for (int j = i + 1; j < 5; ++j)
      if (overlaps(outs[i], outn[i], outs[j], outn[j])) return MHC_ERR_ALIAS;
  }
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  PreBwdArgs a{d_y, d_pre, d_post, d_comb, R, hc_fn, hc_scale, hc_base, d_R, d_hc_fn, d_scale,
               d_base, workspace, T, H, prm.sinkhorn_iters, prm.sinkhorn_eps, prm.rms_eps,
               prm.pre_eps, prm.post_mult};
  return launch_pre_backward(a, reinterpret_cast<cudaStream_t>(stream));
}

int mhc_expand(const uint16_t* hidden, uint16_t* streams, int64_t T, int64_t H,
               mhc_stream_t stream) {
  if (T < 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!hidden || !streams) return MHC_ERR_INVALID_ARG;
  if (overlaps(hidden, static_cast<size_t>(T) * H * 2, streams, static_cast<size_t>(T) * 8 * H))
    return MHC_ERR_ALIAS;
  int st = bind_device(hidden);
  if (st != MHC_OK) return st;
  return launch_expand(hidden, streams, T, H, reinterpret_cast<cudaStream_t>(stream));
}

int mhc_head_mean(const uint16_t* R, uint16_t* y, int64_t T, int64_t H, mhc_stream_t stream) {
  if (T < 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!R || !y) return MHC_ERR_INVALID_ARG;
  if (overlaps(R, static_cast<size_t>(T) * 8 * H, y, static_cast<size_t>(T) * H * 2))
    return MHC_ERR_ALIAS;
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  return launch_head_mean(R, y, T, H, reinterpret_cast<cudaStream_t>(stream));
}

// Workspace of mhc_head: [fn24: 4H x 24 fp32][scale3 + base24][pre, post, comb scratch: T x 24
// fp32][mhc_pre workspace], each part 256-byte aligned.
struct HeadLayout {
  size_t fn, sb, coef, pre_ws, pre_ws_bytes, total;
};
static HeadLayout head_layout(int64_t T, int64_t H) {
  HeadLayout l;
  auto up = [](size_t v) { return (v + 255) / 256 * 256; };
  l.fn = 0;
  l.sb = up(static_cast<size_t>(4 * H) * 24 * 4);
  l.coef = l.sb + 256;
  l.pre_ws = l.coef + up(static_cast<size_t>(T) * 24 * 4);
  l.pre_ws_bytes = mhc_pre_workspace_bytes(T, H);
  l.total = l.pre_ws + l.pre_ws_bytes;
  return l;
}

size_t mhc_head_workspace_bytes(int64_t T, int64_t H) {
  if (T <= 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return 0;
  return head_layout(T, H).total;
}

int mhc_head(const uint16_t* R, const float* hc_fn, const float* hc_scale, const float* hc_base,
             uint16_t* y, float* weights, void* workspace, size_t workspace_bytes, int64_t T,
             int64_t H, float norm_eps, float hc_eps, mhc_stream_t stream) {
  if (T < 0 || H <= 0 || !mul_ok(T, 4 * H, INT64_MAX / 4)) return MHC_ERR_INVALID_ARG;
  if (!(norm_eps > 0.0f) || !isfinite(norm_eps) || !(hc_eps >= 0.0f) || !isfinite(hc_eps))
    return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!R || !hc_fn || !hc_scale || !hc_base || !y) return MHC_ERR_INVALID_ARG;
  const HeadLayout l = head_layout(T, H);
  if (workspace_bytes < l.total || !workspace) return MHC_ERR_WORKSPACE_TOO_SMALL;
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) return MHC_ERR_INVALID_ARG;
  const size_t nR = static_cast<size_t>(T) * 8 * H, ny = static_cast<size_t>(T) * H * 2;
  const size_t nfn = static_cast<size_t>(4 * H) * 16;
  if (overlaps(y, ny, R, nR) || overlaps(y, ny, hc_fn, nfn) || overlaps(y, ny, workspace, l.total))
    return MHC_ERR_ALIAS;
  if (overlaps(workspace, l.total, R, nR) || overlaps(workspace, l.total, hc_fn, nfn))
    return MHC_ERR_ALIAS;
  if (weights && (overlaps(weights, static_cast<size_t>(T) * 16, y, ny) ||
                  overlaps(weights, static_cast<size_t>(T) * 16, R, nR) ||
                  overlaps(weights, static_cast<size_t>(T) * 16, workspace, l.total)))
    return MHC_ERR_ALIAS;
  int st = bind_device(R);
  if (st != MHC_OK) return st;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  float* fn24 = reinterpret_cast<float*>(ws + l.fn);
  float* sb = reinterpret_cast<float*>(ws + l.sb);
  float* coef = reinterpret_cast<float*>(ws + l.coef);
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int r = launch_head_pad(hc_fn, hc_scale, hc_base, fn24, sb, H, s);
  if (r != 0) return r;
  // The pre-map with that padded projection: its pre gates are the head weights; post and comb
  // (one Sinkhorn round) land in scratch.
  mhc_params p;
  p.sinkhorn_iters = 1;
  p.sinkhorn_eps = 1e-6f;
  p.rms_eps = norm_eps;
  p.pre_eps = hc_eps;
  p.post_mult = 1.0f;
  float* pre_out = weights ? weights : coef;
  return mhc_pre_with_path(R, fn24, sb, sb + 3, y, pre_out, coef + 4 * T, coef + 8 * T,
                           ws + l.pre_ws, l.pre_ws_bytes, T, H, &p, MHC_PATH_AUTO, stream);
}

int mhc_selftest_wait_timeout(int64_t limit_ns, mhc_stream_t stream) {
  if (limit_ns < 1000 || limit_ns > 1000000000) return MHC_ERR_INVALID_ARG;
  const int dev = current_device();
  if (dev < 0) return MHC_ERR_CUDA;
  if (device_cc() / 10 != 10) return MHC_ERR_UNSUPPORTED;
  selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<unsigned long long>(limit_ns));
  note_launches(1);
  return cudaGetLastError() == cudaSuccess ? MHC_OK : MHC_ERR_CUDA;
}

int mhc_device_status(mhc_stream_t stream) {
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaStreamSynchronize(s) != cudaSuccess) return MHC_ERR_CUDA;
  int v = 0, zero = 0;
  if (cudaMemcpyFromSymbol(&v, g_device_status, sizeof(int)) != cudaSuccess) return MHC_ERR_CUDA;
  if (cudaMemcpyToSymbol(g_device_status, &zero, sizeof(int)) != cudaSuccess) return MHC_ERR_CUDA;
  return v;
}

}  // extern "C"
