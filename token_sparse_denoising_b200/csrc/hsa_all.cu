// hsa_all.cu -- single translation unit of libhsa.so (the device status word is
// shared by every kernel without relocatable device code).
#include "runtime.cu"
#include "plan.cu"
#include "stream_kernels.cu"
#include "select.cu"
#include "gemm_tc.cu"
#include "attn_tc.cu"
#include "simt_f32.cu"
#include "api.cu"
#include "host_io.cu"
#include "shard.cu"
#include "noalloc.cu"
