#pragma once
// Fused dequant-GEMV / small-M GEMM on CUDA cores (sm_100a).
//
// y[m][o] = sum_i X[m][i] * w_hat[o][i] with w_hat the HLWQ Q5 weights
// ("Qwen3.6-35B-A3B -- HLWQ Q5", Method), evaluated in the rotated domain by
// the decode engine (engine.cuh): the CTA rotates its tokens' activations once
// (FWHT per 128-block, binary16 in shared memory), then every weight costs one
// table lookup and one fp32-accumulating FMA per token.
//
// One persistent CTA of 512 threads per SM (the 128 KiB lane-replicated pair
// table fills most of the SM's shared memory); the O rows are split into equal
// contiguous ranges of whole row groups, one per CTA, so every SM streams the
// same number of code bytes.  Tokens are processed MT (1, 2 or 4) at a time;
// the chunk partial sums are added in a fixed order, so results are
// deterministic.

#include <algorithm>

#include "engine.cuh"

namespace hlwq {

namespace {

template <int C, int MT>
__global__ void __launch_bounds__(kEngineThreads, 1)
dense_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
             const float* __restrict__ codebook, int64_t O, int in, int nb,
             const uint16_t* __restrict__ X, int64_t ldx, int M, void* __restrict__ Y, int64_t ldy,
             int out_bf16, int max_rows) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int G = 32 / C;
  const int nch = (nb + C - 1) / C;
  const EngineLayout L = engine_layout(MT, nb, max_rows, nch);
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* slots = reinterpret_cast<float*>(smem + L.slot_off);
  float* misc = reinterpret_cast<float*>(smem + L.misc_off);
  float* inv_scale = misc + 48;  // [MT] (MT <= 16)
  uint16_t* c16 = reinterpret_cast<uint16_t*>(misc + 64);

  const int64_t ngroups = (O + G - 1) / G;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * ngroups / gridDim.x;
  const int64_t g1 = static_cast<int64_t>(blockIdx.x + 1) * ngroups / gridDim.x;
  const int64_t row0 = g0 * G;
  const int nvrows = static_cast<int>(std::min<int64_t>(g1 * G, O) - row0);

  build_pair_table(tab, c16, codebook);
  for (int m0 = 0; m0 < M; m0 += MT) {
    const int ntok = std::min(MT, M - m0);
    rotate_activations_bf16(X + m0 * ldx, ldx, in, nb, ntok, MT, xs, inv_scale, misc);
    if (nvrows > 0)
      engine_items<C, MT>(tab, xs, packed, norms, nb, nvrows, [&](int v) { return row0 + v; }, slots);
    __syncthreads();
    for (int idx = threadIdx.x; idx < ntok * nvrows; idx += blockDim.x) {
      const int m = idx / nvrows, v = idx - m * nvrows;
      const float* sl = slots + (m * nvrows + v) * nch;
      float sum = 0.0f;
      for (int ch = 0; ch < nch; ++ch) sum += sl[ch];
      sum *= inv_scale[m];
      const int64_t off = (m0 + m) * ldy + row0 + v;
      if (out_bf16) static_cast<uint16_t*>(Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(sum));
      else static_cast<float*>(Y)[off] = sum;
    }
    __syncthreads();
  }
}

template <int C, int MT>
int launch_dense_t(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
                   cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  constexpr int G = 32 / C;
  const int64_t ngroups = ceil_div(O, G);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int max_rows = static_cast<int>(ceil_div(ngroups, grid) * G);
  const int nch = (nb + C - 1) / C;
  const EngineLayout L = engine_layout(MT, nb, max_rows, nch);
  if (L.total > 227 * 1024) return HLWQ_EUNSUPPORTED;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(dense_kernel<C, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
        cudaSuccess)
      return HLWQ_ECUDA;
    attr_set = true;
  }
  dense_kernel<C, MT><<<grid, kEngineThreads, L.total, stream>>>(packed, norms, codebook, O, in, nb, X, ldx, M, Y,
                                                                  ldy, out_bf16 ? 1 : 0, max_rows);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

template <int C>
int launch_dense_c(int mt, const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16,
                   cudaStream_t stream) {
  switch (mt) {
    case 1: return launch_dense_t<C, 1>(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    case 2: return launch_dense_t<C, 2>(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    default: return launch_dense_t<C, 4>(packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
  }
}

}  // namespace

// Shared-memory bytes the dense kernel needs for a given shape and token tile.
int dense_smem_bytes(int64_t O, int in, int mt) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int C = pick_chunk(nb), G = 32 / C;
  const int64_t ngroups = ceil_div(O, G);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int max_rows = static_cast<int>(ceil_div(ngroups, grid) * G);
  return engine_layout(mt, nb, max_rows, (nb + C - 1) / C).total;
}

int launch_dense(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* X, int64_t ldx, int M, void* Y, int64_t ldy, bool out_bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  int mt = M >= 3 ? 4 : M;
  while (mt > 1 && dense_smem_bytes(O, in, mt) > 227 * 1024) mt >>= 1;
  switch (pick_chunk(nb)) {
    case 8: return launch_dense_c<8>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    case 4: return launch_dense_c<4>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    default: return launch_dense_c<2>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
  }
}

}  // namespace hlwq
