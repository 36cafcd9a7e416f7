#pragma once
// Small-M GEMM entry for M >= 16 (placeholder routing to the CUDA-core decode
// path until the tensor-core kernel lands).
#include "hlwq_common.cuh"

namespace hlwq {

int launch_dense(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream);

size_t gemm_tc_workspace_bytes(int64_t, int64_t, int64_t) { return 0; }

int launch_gemm_tc(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, void*, size_t,
                   cudaStream_t stream) {
  return launch_dense(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
}

}  // namespace hlwq
