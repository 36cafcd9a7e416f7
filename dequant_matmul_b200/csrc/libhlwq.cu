// Single translation unit of libhlwq: the kernels share the device error word
// and are compiled together (no relocatable device code needed).
#include "quantize.cuh"
#include "gemv.cuh"
#include "gemvm.cuh"
#include "moe.cuh"
#include "moe1.cuh"
#include "gemm_tc.cuh"
#include "int4.cuh"
#include "kv.cuh"
#include "codes.cuh"
#include "tq3.cuh"
#include "api.cuh"
