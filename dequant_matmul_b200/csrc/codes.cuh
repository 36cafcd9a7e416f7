#pragma once
// One-code-per-byte layout of the HLWQ Q5 codes (sm_100a).
//
// "Gemma-4-26B-A4B-it-HLWQ-Q5", Technical Details: that release stores the
// codes as int8, one code per byte, next to fp16 norms; the canonical form is
// the packed 5-bit stream of "Qwen3.6-35B-A3B -- HLWQ Q5", Method step [5]
// (8 codes in 5 bytes, code j at bits [5j, 5j+5), least significant bit
// first).  These two kernels convert between the layouts:
//   codes  uint8 [nblocks][128], values 0..31
//   packed uint8 [nblocks][80]
// A code above 31 is stored by its low five bits and sets
// HLWQ_DEVERR_CODE_RANGE.
//
// Layout: a warp converts eight blocks per step, four lanes per block and 32
// codes (20 packed bytes) per lane.  The packed side moves through shared
// memory as whole 16-byte words (80 bytes = five of them per block), so both
// sides are read and written with 16-byte accesses; lane l's five packed words
// sit at shared word 5l + k, which keeps the 32 lanes on distinct banks.

#include "hlwq_common.cuh"

namespace hlwq {

namespace {

constexpr int kCodesThreads = 256;
constexpr int kCodesWarps = kCodesThreads / 32;
constexpr int kCodesStepBlocks = 8;                       // blocks per warp step
constexpr int kCodesStepWords = kCodesStepBlocks * 20;    // 32-bit words of packed codes per step

__device__ __forceinline__ void put_step(uint32_t* st, const uint8_t* src, int nv, int lane) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
  uint4* d = reinterpret_cast<uint4*>(st);
  for (int i = lane; i < nv * 5; i += 32) d[i] = ldg_stream(s + i);
}

__global__ void __launch_bounds__(kCodesThreads)
codes_unpack_kernel(const uint8_t* __restrict__ packed, int64_t nblocks, uint8_t* __restrict__ codes) {
  __shared__ __align__(16) uint32_t stage[kCodesWarps][kCodesStepWords];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint32_t* st = stage[wib];
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * kCodesWarps + wib;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kCodesWarps;
  for (int64_t first = warp * kCodesStepBlocks; first < nblocks; first += nwarps * kCodesStepBlocks) {
    const int nv = static_cast<int>(nblocks - first < kCodesStepBlocks ? nblocks - first : kCodesStepBlocks);
    put_step(st, packed + first * kBlockBytes, nv, lane);
    __syncwarp();
    if ((lane >> 2) < nv) {
      uint32_t w[6];
#pragma unroll
      for (int k = 0; k < 5; ++k) w[k] = st[5 * lane + k];
      w[5] = 0u;
      uint32_t out[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) out[k] = 0u;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int bit = 5 * e, k = bit >> 5, sh = bit & 31;
        const uint32_t c = (sh <= 27) ? ((w[k] >> sh) & 31u) : (__funnelshift_r(w[k], w[k + 1], sh) & 31u);
        out[e >> 2] |= c << (8 * (e & 3));
      }
      uint4* dst = reinterpret_cast<uint4*>(codes + (first + (lane >> 2)) * kBlock + 32 * (lane & 3));
      dst[0] = make_uint4(out[0], out[1], out[2], out[3]);
      dst[1] = make_uint4(out[4], out[5], out[6], out[7]);
    }
    __syncwarp();
  }
}

__global__ void __launch_bounds__(kCodesThreads)
codes_pack_kernel(const uint8_t* __restrict__ codes, int64_t nblocks, uint8_t* __restrict__ packed) {
  __shared__ __align__(16) uint32_t stage[kCodesWarps][kCodesStepWords];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  uint32_t* st = stage[wib];
  const int64_t warp = static_cast<int64_t>(blockIdx.x) * kCodesWarps + wib;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * kCodesWarps;
  for (int64_t first = warp * kCodesStepBlocks; first < nblocks; first += nwarps * kCodesStepBlocks) {
    const int nv = static_cast<int>(nblocks - first < kCodesStepBlocks ? nblocks - first : kCodesStepBlocks);
    bool over = false;
    if ((lane >> 2) < nv) {
      const uint4* src = reinterpret_cast<const uint4*>(codes + (first + (lane >> 2)) * kBlock + 32 * (lane & 3));
      const uint4 a = ldg_stream(src), b = ldg_stream(src + 1);
      const uint32_t in[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      uint32_t w[6] = {0u, 0u, 0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const uint32_t raw = (in[e >> 2] >> (8 * (e & 3))) & 0xffu;
        over |= raw > 31u;
        const uint32_t c = raw & 31u;
        const int bit = 5 * e, k = bit >> 5, sh = bit & 31;
        w[k] |= c << sh;
        if (sh > 27) w[k + 1] |= c >> (32 - sh);
      }
#pragma unroll
      for (int k = 0; k < 5; ++k) st[5 * lane + k] = w[k];
    }
    if (__any_sync(0xffffffffu, over) && lane == 0) raise_device_error(HLWQ_DEVERR_CODE_RANGE);
    __syncwarp();
    uint4* d = reinterpret_cast<uint4*>(packed + first * kBlockBytes);
    const uint4* s = reinterpret_cast<const uint4*>(st);
    for (int i = lane; i < nv * 5; i += 32) d[i] = s[i];
    __syncwarp();
  }
}

int codes_grid(int64_t nblocks) {
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 8;
  return static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(nblocks, kCodesWarps * kCodesStepBlocks)));
}

}  // namespace

int launch_codes_unpack(const uint8_t* packed, int64_t nblocks, uint8_t* codes, cudaStream_t stream) {
  codes_unpack_kernel<<<codes_grid(nblocks), kCodesThreads, 0, stream>>>(packed, nblocks, codes);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_codes_pack(const uint8_t* codes, int64_t nblocks, uint8_t* packed, cudaStream_t stream) {
  codes_pack_kernel<<<codes_grid(nblocks), kCodesThreads, 0, stream>>>(codes, nblocks, packed);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace hlwq
