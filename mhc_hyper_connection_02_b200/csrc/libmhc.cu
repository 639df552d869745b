// Single translation unit of libmhc.so: the device status word that bounded waits write
// (mhc::g_device_status, defined in mhc_api.cu) is shared by every kernel without relocatable
// device code.
#include "mhc_api.cu"
#include "mhc_post.cu"
#include "mhc_sinkhorn.cu"
#include "mhc_pre_cc.cu"
#include "mhc_pre_tc.cu"
#include "mhc_pre_fused.cu"
#include "mhc_pre_wave.cu"
#include "mhc_pre_noalloc.cu"
#include "mhc_pre_bigfuse.cu"
#include "mhc_boundary.cu"
#include "mhc_post_project.cu"
#include "mhc_backward.cu"
#include "mhc_backward_tc.cu"
