// moe_boundary.cu -- single translation unit of libmoe_boundary.so.
//
// The kernels share one device-side status word (mb::g_wait_timeout), so the
// library is compiled as one unit instead of relocatable device code.
#include "api.cu"
#include "combine.cu"
#include "route.cu"
#include "norm_quant.cu"
#include "decode.cu"
#include "router_proj.cu"
#include "dispatch.cu"
#include "dispatch_noalloc.cu"
#include "finalize_ar.cu"
