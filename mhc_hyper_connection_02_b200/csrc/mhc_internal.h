// Host-side declarations shared by the library's translation units (not part of the C ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include <cstddef>
#include <utility>

namespace mhc {

// Launches `kernel` on stream s with programmatic stream serialisation: the grid may begin
// launching while the previous grid in the stream finishes; the kernel orders itself behind that
// grid with pdl_wait (mhc_device.cuh) before touching global memory.
template <typename... Params, typename... Args>
cudaError_t launch_pdl(void (*kernel)(Params...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Device of the calling thread (this runtime instance), or -1 on error.
int current_device();
// Streaming multiprocessors of the current device (cached per device).
int device_sm_count();
// Compute capability major*10+minor of the current device (cached per device).
int device_cc();

// Counts kernel launches enqueued through the library (mhc_launch_count).
void note_launches(int n);

// Raises `kernel`'s dynamic shared-memory limit to `bytes` on the current device, once per
// (kernel, device); safe to call from several host threads. Returns false if the runtime refuses.
bool ensure_smem_limit(const void* kernel, int bytes);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// Launchers return 0 or a negative MHC_ERR_* code.
int launch_post_vec8(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                     uint16_t* out, int64_t T, int64_t H, cudaStream_t s);
int launch_post_scalar(const uint16_t* x, const uint16_t* R, const float* post, const float* comb,
                       uint16_t* out, int64_t T, int64_t H, cudaStream_t s);
int launch_post_persistent(const uint16_t* x, const uint16_t* R, const float* post,
                           const float* comb, uint16_t* out, int64_t T, int64_t H,
                           cudaStream_t s);

int launch_sinkhorn(const float* logits, float* comb, int64_t T, int iters, float eps,
                    cudaStream_t s);

struct PreArgs {
  const uint16_t* R;
  const float* hc_fn;
  const float* hc_scale;
  const float* hc_base;
  uint16_t* y;
  float* pre;
  float* post;
  float* comb;
  void* workspace;
  size_t workspace_bytes;
  int64_t T;
  int64_t H;
  int iters;
  float sinkhorn_eps;
  float rms_eps;
  float pre_eps;
  float post_mult;
};

// CUDA-core split-K path.
size_t pre_cc_workspace_bytes(int64_t T, int64_t H);
int launch_pre_cc(const PreArgs& a, cudaStream_t s);
// Its projection step alone: records [nrec][T][32] (raw[24], ss) at the workspace start.
int launch_cc_projection(const PreArgs& a, cudaStream_t s, float** part, int* nrec);

// Tensor-core path: single-pass persistent kernel (launch returns 1, having launched nothing, when
// the device cannot run its grid with every CTA resident).
bool pre_fused_supported(int64_t T, int64_t H);
bool pre_fused_preferred(int64_t T, int64_t H);
size_t pre_fused_workspace_bytes(int64_t T, int64_t H);
int launch_pre_fused(const PreArgs& a, cudaStream_t s);

// Tensor-core path: single pass in wavefront order (mhc_pre_wave.cu; launch returns 1, having
// launched nothing, when the device cannot run its grid with every CTA resident).
bool pre_wave_supported(int64_t T, int64_t H);
size_t pre_wave_workspace_bytes(int64_t T, int64_t H);
int launch_pre_wave(const PreArgs& a, cudaStream_t s);

// Pre-map from an external projection (mhc_pre_big_fuse; sqrsum == nullptr selects the variant
// that forms the sum of squares from R, k = 4H).
struct BigFuseArgs {
  const float* dot_mix;  // [nsplit][T][24]
  const float* sqrsum;   // [nsplit][T] or nullptr
  int nsplit;
  float k;               // RMS denominator
  const uint16_t* R;
  const float* hc_scale;
  const float* hc_base;
  uint16_t* y;
  float* pre;
  float* post;
  float* comb;
  int64_t T;
  int64_t H;
  int iters;
  float sinkhorn_eps;
  float rms_eps;
  float pre_eps;
  float post_mult;
};
int launch_pre_bigfuse(const BigFuseArgs& a, cudaStream_t s);

// Post-map fused with the next site's projection partials (mhc_post_project.cu).
struct PostProjectArgs {
  const uint16_t* x;
  const uint16_t* R;
  const float* post;
  const float* comb;
  uint16_t* out;
  const float* hc_fn;  // the next site's [4H][24]
  float* dot_mix;      // [S][T][24]
  float* sqrsum;       // [S][T]
  void* workspace;
  int64_t T;
  int64_t H;
};
bool post_project_supported(int64_t T, int64_t H);
int post_project_splits(int64_t T, int64_t H);
size_t post_project_workspace_bytes(int64_t T, int64_t H);
int launch_post_project(const PostProjectArgs& a, cudaStream_t s);

// Backward passes (mhc_backward.cu).
int launch_post_backward(const uint16_t* dout, const uint16_t* x, const uint16_t* R,
                         const float* post, const float* comb, uint16_t* dx, uint16_t* dR,
                         float* dpost, float* dcomb, int64_t T, int64_t H, cudaStream_t s);
struct PreBwdArgs {
  const uint16_t* dy;   // [T][H] or null
  const float* dpre;    // [T][4] or null
  const float* dpost;   // [T][4] or null
  const float* dcomb;   // [T][4][4] or null
  const uint16_t* R;
  const float* hc_fn;
  const float* hc_scale;
  const float* hc_base;
  uint16_t* dR;
  float* dW;            // [4H][24]
  float* dscale;        // [3]
  float* dbase;         // [24]
  void* workspace;
  int64_t T;
  int64_t H;
  int iters;
  float sinkhorn_eps;
  float rms_eps;
  float pre_eps;
  float post_mult;
};
size_t pre_backward_workspace_bytes(int64_t T, int64_t H);
// d_R and d_hc_fn of the pre-map backward on tensor cores in one pass over R (mhc_backward_tc.cu):
// 0, a negative MHC_ERR_* code, or 1 when this form cannot run the shape (nothing launched).
bool pre_bwd_dr_tc_supported(int64_t T, int64_t H);
size_t pre_bwd_dr_tc_workspace_bytes(int64_t T, int64_t H);
int launch_pre_bwd_dr_tc(const uint16_t* R, const uint16_t* dy, const float* hc_fn,
                         const float* brec, int rec_stride, uint16_t* dR, float* dW, void* ws,
                         int64_t T, int64_t H, cudaStream_t s);
// d_hc_fn alone on tensor cores (where the fused form cannot run): same return convention.
bool pre_bwd_dw_tc_supported(int64_t T, int64_t H);
size_t pre_bwd_dw_tc_workspace_bytes(int64_t T, int64_t H);
int launch_pre_bwd_dw_tc(const uint16_t* R, const float* brec, int rec_stride, float* dW,
                         void* ws, int64_t T, int64_t H, cudaStream_t s);
int launch_pre_backward(const PreBwdArgs& a, cudaStream_t s);

// Model-boundary operations (mhc_boundary.cu).
int launch_expand(const uint16_t* hidden, uint16_t* streams, int64_t T, int64_t H, cudaStream_t s);
int launch_head_mean(const uint16_t* R, uint16_t* y, int64_t T, int64_t H, cudaStream_t s);
int launch_head_pad(const float* fn4, const float* scale1, const float* base4, float* fn24,
                    float* sb, int64_t H, cudaStream_t s);

// Tensor-core path, split pair (projection kernel + finish kernel).
size_t pre_tc_workspace_bytes(int64_t T, int64_t H);
bool pre_tc_supported(int64_t T, int64_t H);
int launch_pre_tc(const PreArgs& a, cudaStream_t s);
// The tensor path's split + projection alone: records [nrec][T][32] after the Bw operand.
// With dy (the pre-map backward; H % 64 == 0) the records also carry sum_h dy R_i per stream in
// floats 28..31.
int launch_tc_projection(const PreArgs& a, cudaStream_t s, float** part, int* nrec,
                         const uint16_t* dy = nullptr);

}  // namespace mhc
