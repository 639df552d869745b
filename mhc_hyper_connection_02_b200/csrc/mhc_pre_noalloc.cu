// mhc_pre_noalloc: the CUDA-core pre-map with its scratch in a fixed device array owned by the
// library, for callers that cannot allocate device memory (see include/mhc.h).
//
// The scratch is the split-K record buffer [nsplit][T][32] fp32 that the partial kernel writes and
// the finish kernel reads. Every record the finish kernel reads is written first by the partial
// kernel of the same call, so nothing needs clearing between calls. The array is shared by every
// call on a device: calls whose kernels overlap on the GPU (different streams, no ordering between
// them) race on it.
#include "mhc.h"
#include "mhc_device.cuh"
#include "mhc_internal.h"

namespace mhc {

// Loaded with the library's module on every GPU that runs it, and held until the process exits.
static __device__ __align__(256) uint8_t g_noalloc_scratch[MHC_NOALLOC_SCRATCH_BYTES];

namespace {
// Device address of g_noalloc_scratch on the current device. In host code the symbol's name is a
// host-side stand-in, not a device address, so the address is looked up with the device current.
// It is looked up on every call rather than cached: after a device reset or a new context the
// module is loaded again, possibly elsewhere, and a cached address would point at freed memory.
int noalloc_scratch(void** out) {
  void* p = nullptr;
  if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
    cudaGetLastError();
    return MHC_ERR_CUDA;
  }
  *out = p;
  return MHC_OK;
}

bool ranges_overlap(const void* a, size_t na, const void* b, size_t nb) {
  const uintptr_t x = reinterpret_cast<uintptr_t>(a), y = reinterpret_cast<uintptr_t>(b);
  return na > 0 && nb > 0 && x < y + nb && y < x + na;
}
}  // namespace

}  // namespace mhc

extern "C" int mhc_pre_noalloc(const uint16_t* R, const float* hc_fn, const float* hc_scale,
                               const float* hc_base, uint16_t* y, float* pre, float* post,
                               float* comb, int64_t T, int64_t H, const mhc_params* p,
                               mhc_stream_t stream) {
  using namespace mhc;
  const mhc_params prm = p ? *p : mhc_default_params();
  if (T < 0 || H <= 0 || H > (INT64_MAX / 16) || (T > 0 && T > INT64_MAX / (16 * H)))
    return MHC_ERR_INVALID_ARG;
  if (prm.sinkhorn_iters < 1 || !(prm.sinkhorn_eps > 0.0f) || !isfinite(prm.sinkhorn_eps) ||
      !(prm.rms_eps > 0.0f) || !isfinite(prm.rms_eps) || !(prm.pre_eps >= 0.0f) ||
      !isfinite(prm.pre_eps) || !isfinite(prm.post_mult))
    return MHC_ERR_INVALID_ARG;
  if (T == 0) return MHC_OK;
  if (!R || !hc_fn || !hc_scale || !hc_base || !y || !pre || !post || !comb)
    return MHC_ERR_INVALID_ARG;
  if (pre_cc_workspace_bytes(T, H) > MHC_NOALLOC_SCRATCH_BYTES) return MHC_ERR_SCRATCH_LIMIT;
  const size_t nR = static_cast<size_t>(T) * 4 * H * 2, ny = static_cast<size_t>(T) * H * 2;
  const size_t n4 = static_cast<size_t>(T) * 16, n16 = static_cast<size_t>(T) * 64;
  const void* outs[4] = {y, pre, post, comb};
  const size_t outn[4] = {ny, n4, n4, n16};
  const void* ins[4] = {R, hc_fn, hc_scale, hc_base};
  const size_t inn[4] = {nR, static_cast<size_t>(H) * 4 * 24 * 4, 12, 96};
  for (int i = 0; i < 4; ++i) {
    for (int j = 0; j < 4; ++j)
      if (ranges_overlap(outs[i], outn[i], ins[j], inn[j])) return MHC_ERR_ALIAS;
    for (int j = i + 1; j < 4; ++j)
      if (ranges_overlap(outs[i], outn[i], outs[j], outn[j])) return MHC_ERR_ALIAS;
  }
  // Bind this runtime to the device that owns R (and check it is device memory on an sm_100).
  cudaPointerAttributes at;
  if (cudaPointerGetAttributes(&at, R) != cudaSuccess) {
    cudaGetLastError();
    return MHC_ERR_INVALID_ARG;
  }
  if (at.type != cudaMemoryTypeDevice && at.type != cudaMemoryTypeManaged) return MHC_ERR_INVALID_ARG;
  int cur = -1;
  if (cudaGetDevice(&cur) != cudaSuccess) return MHC_ERR_CUDA;
  if (cur != at.device && cudaSetDevice(at.device) != cudaSuccess) return MHC_ERR_CUDA;
  if (device_cc() / 10 != 10) return MHC_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  const int st = noalloc_scratch(&scratch);
  if (st != MHC_OK) return st;
  PreArgs a{R, hc_fn, hc_scale, hc_base, y, pre, post, comb, scratch, MHC_NOALLOC_SCRATCH_BYTES,
            T, H, prm.sinkhorn_iters, prm.sinkhorn_eps, prm.rms_eps, prm.pre_eps, prm.post_mult};
  return launch_pre_cc(a, reinterpret_cast<cudaStream_t>(stream));
}
