// mHC pre-map on tcgen05 tensor cores (placeholder until the fused kernel lands).
#include "mhc_internal.h"

namespace mhc {

size_t pre_tc_workspace_bytes(int64_t, int64_t) { return 0; }
bool pre_tc_supported(int64_t, int64_t) { return false; }
int launch_pre_tc(const PreArgs&, cudaStream_t) { return -5; }

}  // namespace mhc
