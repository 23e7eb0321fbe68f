// Single translation unit of libmhc: the kernels share a few device globals
// (the bounded-wait error word and limit), so they are compiled together.
#include "api.cu"
#include "mhc_post.cu"
#include "mhc_pre_fma.cu"
#include "mhc_pre_tc.cu"
#include "mhc_pre_wide.cu"
#include "xhc_conv_gs.cu"
#include "xhc_update.cu"
#include "xhc_update_tc.cu"
#include "xhc_route.cu"
#include "xhc_route_tc.cu"
#include "mhc_bwd.cu"
#include "mhc_bwd_noalloc.cu"
