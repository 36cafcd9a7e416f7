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
  float* xinv = reinterpret_cast<float*>(smem + L.xinv_off);
  float* slots = reinterpret_cast<float*>(smem + L.slot_off);
  float* misc = reinterpret_cast<float*>(smem + L.misc_off);
  uint16_t* c16 = reinterpret_cast<uint16_t*>(misc + 64);

  const int64_t ngroups = (O + G - 1) / G;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * ngroups / gridDim.x;
  const int64_t g1 = static_cast<int64_t>(blockIdx.x + 1) * ngroups / gridDim.x;
  const int64_t row0 = g0 * G;
  const int nvrows = static_cast<int>(std::min<int64_t>(g1 * G, O) - row0);
  auto rowfn = [=](int v) { return row0 + v; };

  for (int m0 = 0; m0 < M; m0 += MT) {
    const int ntok = std::min(MT, M - m0);
    auto eng = make_engine<C, MT>(packed, norms, nb, nvrows, rowfn);
    eng.prefetch();  // code loads in flight while the tables and activations are prepared
    if (m0 == 0) build_pair_table(tab, c16, codebook);
    rotate_tokens_bf16(X + m0 * ldx, ldx, in, nb, ntok, MT, xs, xinv);
    __syncthreads();
    eng.run(tab, xs, xinv, slots);
    __syncthreads();
    for (int idx = threadIdx.x; idx < ntok * nvrows; idx += blockDim.x) {
      const int m = idx / nvrows, v = idx - m * nvrows;
      const float* sl = slots + (m * nvrows + v) * nch;
      float sum = 0.0f;
      for (int ch = 0; ch < nch; ++ch) sum += sl[ch];
      const int64_t off = (m0 + m) * ldy + row0 + v;
      if (out_bf16) static_cast<uint16_t*>(Y)[off] = static_cast<uint16_t>(float_to_bf16_bits(sum));
      else static_cast<float*>(Y)[off] = sum;
    }
    __syncthreads();
  }
}


// Single-token GEMV.  512 threads (16 warps) per CTA, one CTA per SM (the
// 128 KiB pair table).  A lane owns half a 128-block (64 codes, 40 bytes): lane
// (r, s, h) takes row r, block s of the chunk and half h, so the 2C lanes of a
// row read 80 C contiguous bytes.  A CTA's items are ordered chunk-major and
// each warp takes a contiguous range of them, so a lane's 64 rotated
// activation values (32 half2 registers) are reloaded only when the range
// crosses into the next chunk.
constexpr int kGemv1Threads = 512;
constexpr int kGemv1Warps = kGemv1Threads / 32;

template <int C>
__global__ void __launch_bounds__(kGemv1Threads, 1)
gemv1_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
             const float* __restrict__ codebook, int64_t O, int in, int nb, const uint16_t* __restrict__ x,
             void* __restrict__ Y, int out_bf16, int max_rows) {
  extern __shared__ __align__(16) uint8_t smem[];
  constexpr int L2C = 2 * C;      // lanes per row
  constexpr int G = 32 / L2C;     // rows per item
  constexpr int kDepth = 3;
  const int nch = (nb + C - 1) / C;
  const EngineLayout L = engine_layout(1, nb, max_rows, nch);
  uint32_t* tab = reinterpret_cast<uint32_t*>(smem);
  uint16_t* xs = reinterpret_cast<uint16_t*>(smem + L.xs_off);
  float* xinv = reinterpret_cast<float*>(smem + L.xinv_off);
  float* slots = reinterpret_cast<float*>(smem + L.slot_off);
  float* misc = reinterpret_cast<float*>(smem + L.misc_off);
  uint16_t* c16 = reinterpret_cast<uint16_t*>(misc + 64);

  const int64_t ngroups = (O + G - 1) / G;
  const int64_t g0 = static_cast<int64_t>(blockIdx.x) * ngroups / gridDim.x;
  const int64_t g1 = static_cast<int64_t>(blockIdx.x + 1) * ngroups / gridDim.x;
  const int64_t row0 = g0 * G;
  const int nvrows = static_cast<int>(std::min<int64_t>(g1 * G, O) - row0);
  const int ngr = (nvrows + G - 1) / G;
  const int nitems = ngr * nch;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int r = lane / L2C, u = lane % L2C, s = u >> 1, hh = u & 1;
  const int it0 = warp * nitems / kGemv1Warps, it1 = (warp + 1) * nitems / kGemv1Warps;

  uint2 cw[kDepth][5];
  float sc[kDepth];
  bool ok[kDepth];
  auto fetch = [&](int it, int d) {
    ok[d] = false;
    sc[d] = 0.0f;
    if (it >= it1) return;
    const int ch = it / ngr, g = it - ch * ngr;
    const int vrow = g * G + r, b = ch * C + s;
    if (vrow < nvrows && b < nb) {
      const int64_t F = (row0 + vrow) * nb + b;
      const uint2* src = reinterpret_cast<const uint2*>(packed + F * kBlockBytes + 40 * hh);
#pragma unroll
      for (int q = 0; q < 5; ++q) cw[d][q] = __ldg(src + q);
      sc[d] = half_bits_to_float(__ldg(norms + F)) * (1.0f / 128.0f);
      ok[d] = true;
    }
  };
#pragma unroll
  for (int d = 0; d < kDepth; ++d) fetch(it0 + d, d);  // code loads in flight during the set-up below

  // Set-up, split over the warps: rotate x (four lanes per block) on some
  // warps while the others replicate the pair table.
  load_codebook16(c16, codebook);
  __syncthreads();
  const int nrot = min(kGemv1Warps / 2, (nb + 7) / 8);
  rotate_row_q4(x, in, nb, xs, xinv, 0, nrot);
  build_pair_table_warps(tab, c16, nrot, kGemv1Warps - nrot);
  __syncthreads();

  const uint32_t lane_base = static_cast<uint32_t>(__cvta_generic_to_shared(tab)) + 4u * lane;
  uint32_t xr[32];
  float xi = 0.0f;
  int cur_ch = -1;
  int ch_base = it0 / ngr, g_base = it0 - (it0 / ngr) * ngr;  // (chunk, group) of item `base`
  for (int base = it0; base < it1; base += kDepth) {
#pragma unroll
    for (int d = 0; d < kDepth; ++d) {
      const int it = base + d;
      int ch = ch_base, g = g_base + d;
      if (g >= ngr) { g -= ngr; ++ch; }
      if (g >= ngr) { g -= ngr; ++ch; }
      if (it < it1) {
        const int b = ch * C + s;
        if (ch != cur_ch) {
          cur_ch = ch;
          if (b < nb) {
            const uint4* xsrc = reinterpret_cast<const uint4*>(xs + b * kXsStride + 64 * hh);
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              const uint4 v = xsrc[q];
              xr[4 * q] = v.x; xr[4 * q + 1] = v.y; xr[4 * q + 2] = v.z; xr[4 * q + 3] = v.w;
            }
            xi = xinv[b];
          }
        }
        float acc = ok[d] ? half_dot_reg(cw[d], lane_base, xr) * (sc[d] * xi) : 0.0f;
#pragma unroll
        for (int off = L2C / 2; off > 0; off >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, off);
        const int vrow = g * G + r;
        if (u == 0 && vrow < nvrows) slots[vrow * nch + ch] = acc;
        fetch(it + kDepth, d);
      }
    }
    g_base += kDepth;
    while (g_base >= ngr) { g_base -= ngr; ++ch_base; }
  }
  __syncthreads();
  for (int v = threadIdx.x; v < nvrows; v += blockDim.x) {
    const float* sl = slots + v * nch;
    float sum = 0.0f;
    for (int ch = 0; ch < nch; ++ch) sum += sl[ch];
    if (out_bf16) static_cast<uint16_t*>(Y)[row0 + v] = static_cast<uint16_t>(float_to_bf16_bits(sum));
    else static_cast<float*>(Y)[row0 + v] = sum;
  }
}

template <int C>
int launch_gemv1_c(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                   const uint16_t* x, void* Y, bool out_bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  constexpr int G = 32 / (2 * C);
  const int64_t ngroups = ceil_div(O, G);
  const int grid = static_cast<int>(std::min<int64_t>(sm_count(), ngroups));
  const int max_rows = static_cast<int>(ceil_div(ngroups, grid) * G);
  const EngineLayout L = engine_layout(1, nb, max_rows, (nb + C - 1) / C);
  if (L.total > 227 * 1024) return HLWQ_EUNSUPPORTED;
  static bool attr_set = false;
  if (!attr_set) {
    if (cudaFuncSetAttribute(gemv1_kernel<C>, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
        cudaSuccess)
      return HLWQ_ECUDA;
    attr_set = true;
  }
  gemv1_kernel<C><<<grid, kGemv1Threads, L.total, stream>>>(packed, norms, codebook, O, in, nb, x, Y,
                                                           out_bf16 ? 1 : 0, max_rows);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace

int launch_gemv1(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t O, int in,
                 const uint16_t* x, void* Y, bool out_bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  switch (pick_chunk(nb)) {
    case 8: return launch_gemv1_c<8>(packed, norms, codebook, O, in, x, Y, out_bf16, stream);
    case 4: return launch_gemv1_c<4>(packed, norms, codebook, O, in, x, Y, out_bf16, stream);
    default: return launch_gemv1_c<2>(packed, norms, codebook, O, in, x, Y, out_bf16, stream);
  }
}

namespace {

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
  if (M == 1) return launch_gemv1(packed, norms, codebook, O, in, X, Y, out_bf16, stream);
  int mt = M >= 3 ? 4 : M;
  while (mt > 1 && dense_smem_bytes(O, in, mt) > 227 * 1024) mt >>= 1;
  switch (pick_chunk(nb)) {
    case 8: return launch_dense_c<8>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    case 4: return launch_dense_c<4>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
    default: return launch_dense_c<2>(mt, packed, norms, codebook, O, in, X, ldx, M, Y, ldy, out_bf16, stream);
  }
}

}  // namespace hlwq
