// Single translation unit of libmoge.so: every kernel source and the C ABI.
#include "router.cu"
#include "rows.cu"
#include "gemm_f32.cu"
#include "gemm_tc.cu"
#include "gemm_fp8.cu"
#include "selftest.cu"
#include "api.cu"
#include "route_noalloc.cu"
