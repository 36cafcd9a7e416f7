// Decode engine shared by the fused GEMV / small-M GEMM / routed-MoE kernels.
//
// The product y[m][o] = sum_i x[m][i] w_hat[o][i] is evaluated in the rotated
// domain (H symmetric, H H = 128 I, "Qwen3.6-35B-A3B -- HLWQ Q5", Method
// step [3]):
//     y[m][o] = sum_b (n16[o][b] / 128) * sum_j c[k_obj] * x_tilde[m][128 b + j],
//     x_tilde_b = x_b @ H  (activation rotated once per call),
// so no weight is ever inverse-rotated and each weight costs one table lookup
// and one fused multiply-add per token.
//
// Work decomposition.  A CTA owns a range of "virtual rows" (a caller-supplied
// map turns them into matrix rows).  A warp works on items = (group of G = 32/C
// rows) x (chunk of C consecutive 128-blocks); lane (r, s) = (lane / C,
// lane % C) takes row r and block s of the item, so the C lanes of one row read
// C * 80 contiguous bytes of codes.  Items are spread over the 16 warps; each
// item's per-row partial sum is reduced over the C lanes with shuffles and
// stored into a slot[token][row][chunk] array in shared memory; the caller's
// epilogue sums the chunks in a fixed order (deterministic, no atomics).
//
// Decode.  Codes are read as 5 x 16-byte loads per (row, block).  A pair of
// consecutive codes (10 bits) indexes a 1024-entry table of binary16 pairs
// (c[k0], c[k1]); the table is replicated once per lane so that lane l always
// reads bank l (conflict-free whatever the codes), i.e. one shared-memory
// wavefront decodes 64 weights.  The rotated activation is stored as binary16
// (scaled by a power of two per token to stay in range) and the products are
// accumulated in fp32 with the mixed-precision fma.rn.f32.f16 (exact product).
#pragma once

#include "hlwq_common.cuh"

namespace hlwq {

constexpr int kEngineThreads = 512;
constexpr int kEngineWarps = kEngineThreads / 32;
constexpr int kPairTabBytes = 1024 * 32 * 4;  // 128 KiB
constexpr int kXsStride = 136;                 // halves per rotated block (128 + 8 pad: 272 B)

// Shared-memory layout helpers ------------------------------------------------
struct EngineLayout {
  int xs_off;     // byte offset of the rotated activations [MT][NB][kXsStride] halves
  int slot_off;   // byte offset of slots [MT][rows][nch] floats
  int misc_off;   // byte offset of 64 floats of scratch (scales, reductions)
  int total;      // bytes
};

__host__ __device__ inline EngineLayout engine_layout(int mt, int nb, int rows, int nch) {
  EngineLayout L;
  L.xs_off = kPairTabBytes;
  const int xs_bytes = mt * nb * kXsStride * 2;
  L.slot_off = L.xs_off + ((xs_bytes + 15) & ~15);
  const int slot_bytes = mt * rows * nch * 4;
  L.misc_off = L.slot_off + ((slot_bytes + 15) & ~15);
  L.total = L.misc_off + 64 * 4 + 64;  // + 32 halves of codebook
  return L;
}

// word (v * 32 + lane) = half2(c[v & 31], c[v >> 5]) for every lane.
__device__ __forceinline__ void build_pair_table(uint32_t* tab, uint16_t* c16, const float* __restrict__ codebook) {
  if (threadIdx.x < kLevels) {
    const float c = __ldg(codebook + threadIdx.x);
    c16[threadIdx.x] = __half_as_ushort(__float2half_rn(c));
    if (threadIdx.x + 1 < kLevels && !(c < __ldg(codebook + threadIdx.x + 1))) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
  __syncthreads();
  uint4* t4 = reinterpret_cast<uint4*>(tab);
  for (int q = threadIdx.x; q < 1024 * 8; q += blockDim.x) {
    const int v = q >> 3;  // 8 uint4 (32 words) per table entry
    const uint32_t e = static_cast<uint32_t>(c16[v & 31]) | (static_cast<uint32_t>(c16[v >> 5]) << 16);
    t4[q] = make_uint4(e, e, e, e);
  }
}

// Rotates `ntok` activation rows (bf16, row pitch ldx, length in) into xs as
// binary16 scaled by 2^k (k per token, chosen from max|x| so that
// |x_tilde| <= 128 max|x| 2^k < 2^15); writes 2^-k into inv_scale[m].
// Tokens m >= ntok are zero-filled.  Must be called by the whole CTA.
__device__ __forceinline__ void rotate_activations_bf16(const uint16_t* __restrict__ X, int64_t ldx, int in, int nb,
                                                        int ntok, int mt, uint16_t* xs, float* inv_scale,
                                                        float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int m = 0; m < mt; ++m) {
    float mx = 0.0f;
    if (m < ntok)
      for (int i = threadIdx.x; i < in; i += blockDim.x) mx = fmaxf(mx, fabsf(bf16_bits_to_float(__ldg(X + m * ldx + i))));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.0f;
      for (int w = 0; w < nwarps; ++w) t = fmaxf(t, red[w]);
      int e = 0;
      if (t > 0.0f && isfinite(t)) frexpf(t, &e);
      const int k = max(-120, min(120, 8 - e));
      red[32] = ldexpf(1.0f, k);
      inv_scale[m] = ldexpf(1.0f, -k);
    }
    __syncthreads();
    const float sc = red[32];
    for (int b = warp; b < nb; b += nwarps) {
      float e4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = kBlock * b + 4 * lane + k;
        e4[k] = (m < ntok && i < in) ? bf16_bits_to_float(__ldg(X + m * ldx + i)) : 0.0f;
      }
      float a = e4[0] + e4[1], bb = e4[0] - e4[1], c = e4[2] + e4[3], d = e4[2] - e4[3];
      e4[0] = a + c; e4[1] = bb + d; e4[2] = a - c; e4[3] = bb - d;
#pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float p = __shfl_xor_sync(0xffffffffu, e4[k], h);
          e4[k] = (lane & h) ? p - e4[k] : e4[k] + p;
        }
      }
      const uint32_t lo = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[0] * sc))) |
                          (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[1] * sc))) << 16);
      const uint32_t hi = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[2] * sc))) |
                          (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[3] * sc))) << 16);
      *reinterpret_cast<uint2*>(xs + (m * nb + b) * kXsStride + 4 * lane) = make_uint2(lo, hi);
    }
    __syncthreads();
  }
}

// Same as above for fp32 source rows (the MoE intermediate h), ntok rows given
// by a row-pointer function.
template <typename RowPtr>
__device__ __forceinline__ void rotate_activations_f32(RowPtr rowptr, int in, int nb, int ntok, int mt, uint16_t* xs,
                                                       float* inv_scale, float* red) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int m = 0; m < mt; ++m) {
    const float* src = m < ntok ? rowptr(m) : nullptr;
    float mx = 0.0f;
    if (src)
      for (int i = threadIdx.x; i < in; i += blockDim.x) mx = fmaxf(mx, fabsf(src[i]));
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    if (lane == 0) red[warp] = mx;
    __syncthreads();
    if (threadIdx.x == 0) {
      float t = 0.0f;
      for (int w = 0; w < nwarps; ++w) t = fmaxf(t, red[w]);
      int e = 0;
      if (t > 0.0f && isfinite(t)) frexpf(t, &e);
      const int k = max(-120, min(120, 8 - e));
      red[32] = ldexpf(1.0f, k);
      inv_scale[m] = ldexpf(1.0f, -k);
    }
    __syncthreads();
    const float sc = red[32];
    for (int b = warp; b < nb; b += nwarps) {
      float e4[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const int i = kBlock * b + 4 * lane + k;
        e4[k] = (src && i < in) ? src[i] : 0.0f;
      }
      float a = e4[0] + e4[1], bb = e4[0] - e4[1], c = e4[2] + e4[3], d = e4[2] - e4[3];
      e4[0] = a + c; e4[1] = bb + d; e4[2] = a - c; e4[3] = bb - d;
#pragma unroll
      for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const float p = __shfl_xor_sync(0xffffffffu, e4[k], h);
          e4[k] = (lane & h) ? p - e4[k] : e4[k] + p;
        }
      }
      const uint32_t lo = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[0] * sc))) |
                          (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[1] * sc))) << 16);
      const uint32_t hi = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[2] * sc))) |
                          (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[3] * sc))) << 16);
      *reinterpret_cast<uint2*>(xs + (m * nb + b) * kXsStride + 4 * lane) = make_uint2(lo, hi);
    }
    __syncthreads();
  }
}

__device__ __forceinline__ uint32_t word_of(const uint4 (&c)[5], int i) {
  const uint4 u = c[i >> 2];
  switch (i & 3) {
    case 0: return u.x;
    case 1: return u.y;
    case 2: return u.z;
    default: return u.w;
  }
}

__device__ __forceinline__ uint32_t comp_of(const uint4& u, int t) {
  switch (t) {
    case 0: return u.x;
    case 1: return u.y;
    case 2: return u.z;
    default: return u.w;
  }
}

// Dot products of one (row, block) of codes with MT rotated activation blocks.
template <int MT>
__device__ __forceinline__ void block_dot(const uint4 (&cw)[5], const uint32_t* __restrict__ tab_lane,
                                          const uint16_t* __restrict__ xb, int xs_tok_stride, float (&acc)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
#pragma unroll
  for (int q = 0; q < 16; ++q) {
    uint4 xv[MT];
#pragma unroll
    for (int m = 0; m < MT; ++m) xv[m] = *reinterpret_cast<const uint4*>(xb + m * xs_tok_stride + 8 * q);
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int bit = 40 * q + 10 * t, wi = bit >> 5, sh = bit & 31;
      const uint32_t lo = word_of(cw, wi);
      const uint32_t hi = (wi + 1 < 20) ? word_of(cw, wi + 1) : 0u;
      const uint32_t v10 = (sh <= 22) ? ((lo >> sh) & 0x3ffu) : (__funnelshift_r(lo, hi, sh) & 0x3ffu);
      const uint32_t ent = tab_lane[v10 << 5];
      const uint16_t c0 = static_cast<uint16_t>(ent & 0xffffu), c1 = static_cast<uint16_t>(ent >> 16);
#pragma unroll
      for (int m = 0; m < MT; ++m) {
        const uint32_t xx = comp_of(xv[m], t);
        acc[m] = fma_f16_f32(c0, static_cast<uint16_t>(xx & 0xffffu), acc[m]);
        acc[m] = fma_f16_f32(c1, static_cast<uint16_t>(xx >> 16), acc[m]);
      }
    }
  }
}

// Processes all items of a CTA's virtual-row range.  rowfn(vrow) returns the
// matrix row (index into packed/norms) of a virtual row.  Results go to
// slots[m][vrow][chunk] (MT tokens, scale n16/128 applied, activation scale not).
template <int C, int MT, typename RowFn>
__device__ __forceinline__ void engine_items(const uint32_t* __restrict__ tab, const uint16_t* __restrict__ xs,
                                             const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                                             int nb, int nvrows, RowFn rowfn, float* __restrict__ slots) {
  constexpr int G = 32 / C;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int r = lane / C, s = lane % C;
  const int nch = (nb + C - 1) / C;
  const int ngroups = (nvrows + G - 1) / G;
  const int nitems = ngroups * nch;
  const uint32_t* tab_lane = tab + lane;
  const int xs_tok_stride = nb * kXsStride;

  auto fetch = [&](int it, uint4 (&cw)[5], float& scale, bool& valid) {
    valid = false;
    scale = 0.0f;
    if (it >= nitems) return;
    const int g = it / nch, ch = it - g * nch;
    const int vrow = g * G + r, b = ch * C + s;
    if (vrow < nvrows && b < nb) {
      const int64_t F = rowfn(vrow) * static_cast<int64_t>(nb) + b;
      const uint4* src = reinterpret_cast<const uint4*>(packed + F * kBlockBytes);
#pragma unroll
      for (int q = 0; q < 5; ++q) cw[q] = ldg_stream(src + q);
      scale = half_bits_to_float(__ldg(norms + F)) * (1.0f / 128.0f);
      valid = true;
    }
  };

  uint4 cur[5];
  float cur_scale;
  bool cur_valid;
  int it = warp;
  fetch(it, cur, cur_scale, cur_valid);
  for (; it < nitems; it += kEngineWarps) {
    uint4 nxt[5];
    float nxt_scale;
    bool nxt_valid;
    fetch(it + kEngineWarps, nxt, nxt_scale, nxt_valid);

    const int g = it / nch, ch = it - g * nch;
    const int b = ch * C + s;
    float acc[MT];
    if (cur_valid) {
      block_dot<MT>(cur, tab_lane, xs + b * kXsStride, xs_tok_stride, acc);
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] *= cur_scale;
    } else {
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
    }
#pragma unroll
    for (int m = 0; m < MT; ++m) {
#pragma unroll
      for (int off = C / 2; off > 0; off >>= 1) acc[m] += __shfl_xor_sync(0xffffffffu, acc[m], off);
    }
    const int vrow = g * G + r;
    if (s == 0 && vrow < nvrows) {
#pragma unroll
      for (int m = 0; m < MT; ++m) slots[(m * nvrows + vrow) * nch + ch] = acc[m];
    }
#pragma unroll
    for (int q = 0; q < 5; ++q) cur[q] = nxt[q];
    cur_scale = nxt_scale;
    cur_valid = nxt_valid;
  }
}

// Picks the chunk width C (blocks per item) for a row of nb blocks: the largest
// of 8/4/2 whose padding waste is minimal.
__host__ __device__ inline int pick_chunk(int nb) {
  int best = 8, best_waste = 1 << 30;
  for (int c = 8; c >= 2; c >>= 1) {
    const int waste = ((nb + c - 1) / c) * c - nb;
    if (waste < best_waste) { best = c; best_waste = waste; }
  }
  return best;
}

}  // namespace hlwq
