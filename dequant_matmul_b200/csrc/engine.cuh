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
// wavefront decodes 64 weights.  The rotated activation is stored as binary16,
// scaled by a power of two per 128-block; every product of a binary16
// centroid and a binary16 activation (exact in fp32) is added to an fp32
// accumulator with the mixed-precision FMA.
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
  int xinv_off;   // byte offset of the per-block activation scales [MT][NB] floats
  int slot_off;   // byte offset of slots [MT][rows][nch] floats
  int misc_off;   // byte offset of 64 floats of scratch (scales, reductions)
  int total;      // bytes
};

__host__ __device__ inline EngineLayout engine_layout(int mt, int nb, int rows, int nch) {
  EngineLayout L;
  L.xs_off = kPairTabBytes;
  const int xs_bytes = mt * nb * kXsStride * 2;
  L.xinv_off = L.xs_off + ((xs_bytes + 15) & ~15);
  L.slot_off = L.xinv_off + ((mt * nb * 4 + 15) & ~15);
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

__device__ __forceinline__ uint32_t pack_half2(float lo, float hi) {
  return static_cast<uint32_t>(__half_as_ushort(__float2half_rn(lo))) |
         (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(hi))) << 16);
}

// Rotates one 128-block held 4 values per lane (x_b @ H, Sylvester order:
// butterflies over the lane's 4 values, then over lanes with shuffles), picks
// a power-of-two scale 2^k so that max|x_tilde| * 2^k lies in [2^9, 2^10) (so
// that sums of a few centroid x activation products stay far below the
// binary16 maximum),
// and stores the block as binary16 at dst (4 halves per lane).  Returns 2^-k.
__device__ __forceinline__ float rotate_block_store(float (&e4)[4], uint16_t* dst) {
  const int lane = threadIdx.x & 31;
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
  float mx = fmaxf(fmaxf(fabsf(e4[0]), fabsf(e4[1])), fmaxf(fabsf(e4[2]), fabsf(e4[3])));
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  int e = 0;
  if (mx > 0.0f && isfinite(mx)) frexpf(mx, &e);
  const int k = max(-120, min(120, 10 - e));
  const float sc = ldexpf(1.0f, k);
  const uint32_t lo = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[0] * sc))) |
                      (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[1] * sc))) << 16);
  const uint32_t hi = static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[2] * sc))) |
                      (static_cast<uint32_t>(__half_as_ushort(__float2half_rn(e4[3] * sc))) << 16);
  *reinterpret_cast<uint2*>(dst + 4 * lane) = make_uint2(lo, hi);
  return ldexpf(1.0f, -k);
}

// Rotated activations of `mt` token rows (bf16, pitch ldx, `ntok` real rows,
// the rest zero) into xs[m][b][kXsStride] (binary16) and inv_scale[m * nb + b].
// Work is spread over the CTA's warps; no CTA barrier inside (the caller syncs).
__device__ __forceinline__ void rotate_tokens_bf16(const uint16_t* __restrict__ X, int64_t ldx, int in, int nb,
                                                   int ntok, int mt, uint16_t* xs, float* inv_scale) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int q = warp; q < mt * nb; q += nwarps) {
    const int m = q / nb, b = q - m * nb;
    float e4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = kBlock * b + 4 * lane + k;
      e4[k] = (m < ntok && i < in) ? bf16_bits_to_float(__ldg(X + m * ldx + i)) : 0.0f;
    }
    const float inv = rotate_block_store(e4, xs + (m * nb + b) * kXsStride);
    if (lane == 0) inv_scale[m * nb + b] = inv;
  }
}

// Rotation with four lanes per 128-block (32 consecutive values per lane: five
// butterfly stages in registers, two across the block's lanes).  Warps
// [w0, w0 + nw) of the CTA take part; each covers 8 blocks per step.  The
// block's values are scaled by a power of two so that max |x_tilde| lies in
// [2^9, 2^10) and stored as binary16; the inverse scale goes to inv_scale[b].
__device__ __forceinline__ void rotate_row_q4(const uint16_t* __restrict__ X, int in, int nb, uint16_t* xs,
                                              float* inv_scale, int w0, int nw) {
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, q = lane & 3;
  if (warp < w0 || warp >= w0 + nw) return;
  for (int bb = (warp - w0) * 8; bb < nb; bb += nw * 8) {
    const int b = bb + (lane >> 2);
    const bool act = b < nb;
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int i = kBlock * b + 32 * q + e;
      v[e] = (act && i < in) ? bf16_bits_to_float(__ldg(X + i)) : 0.0f;
    }
#pragma unroll
    for (int h = 1; h < 32; h <<= 1) {
#pragma unroll
      for (int i = 0; i < 32; ++i)
        if ((i & h) == 0) {
          const float a = v[i], c = v[i + h];
          v[i] = a + c;
          v[i + h] = a - c;
        }
    }
#pragma unroll
    for (int lm = 1; lm <= 2; lm <<= 1) {
      const float sgn = (lane & lm) ? -1.0f : 1.0f;
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = fmaf(v[i], sgn, __shfl_xor_sync(0xffffffffu, v[i], lm));
    }
    float mx = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) mx = fmaxf(mx, fabsf(v[i]));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
    int ex = 0;
    if (mx > 0.0f && isfinite(mx)) frexpf(mx, &ex);
    const int k = max(-120, min(120, 10 - ex));
    const float sc = ldexpf(1.0f, k);
    if (act) {
      uint4* dst = reinterpret_cast<uint4*>(xs + b * kXsStride + 32 * q);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = pack_half2(v[8 * c] * sc, v[8 * c + 1] * sc);
        u.y = pack_half2(v[8 * c + 2] * sc, v[8 * c + 3] * sc);
        u.z = pack_half2(v[8 * c + 4] * sc, v[8 * c + 5] * sc);
        u.w = pack_half2(v[8 * c + 6] * sc, v[8 * c + 7] * sc);
        dst[c] = u;
      }
      if (q == 0) inv_scale[b] = ldexpf(1.0f, -k);
    }
  }
}

// Pair table build by warps [w0, w0 + nw) only (see build_pair_table).
__device__ __forceinline__ void build_pair_table_warps(uint32_t* tab, const uint16_t* c16, int w0, int nw) {
  const int warp = threadIdx.x >> 5;
  if (warp < w0 || warp >= w0 + nw) return;
  uint4* t4 = reinterpret_cast<uint4*>(tab);
  for (int q = (warp - w0) * 32 + (threadIdx.x & 31); q < 1024 * 8; q += nw * 32) {
    const int v = q >> 3;
    const uint32_t e = static_cast<uint32_t>(c16[v & 31]) | (static_cast<uint32_t>(c16[v >> 5]) << 16);
    t4[q] = make_uint4(e, e, e, e);
  }
}

__device__ __forceinline__ void load_codebook16(uint16_t* c16, const float* __restrict__ codebook) {
  if (threadIdx.x < kLevels) {
    const float c = __ldg(codebook + threadIdx.x);
    c16[threadIdx.x] = __half_as_ushort(__float2half_rn(c));
    if (threadIdx.x + 1 < kLevels && !(c < __ldg(codebook + threadIdx.x + 1))) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
}

// Same for fp32 source rows given by rowptr(m) (the MoE intermediate h).
template <typename RowPtr>
__device__ __forceinline__ void rotate_tokens_f32(RowPtr rowptr, int in, int nb, int ntok, int mt, uint16_t* xs,
                                                  float* inv_scale) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nwarps = blockDim.x >> 5;
  for (int q = warp; q < mt * nb; q += nwarps) {
    const int m = q / nb, b = q - m * nb;
    const float* src = m < ntok ? rowptr(m) : nullptr;
    float e4[4];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int i = kBlock * b + 4 * lane + k;
      e4[k] = (src && i < in) ? src[i] : 0.0f;
    }
    const float inv = rotate_block_store(e4, xs + (m * nb + b) * kXsStride);
    if (lane == 0) inv_scale[m * nb + b] = inv;
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

__device__ __forceinline__ uint32_t lds_u32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(addr));
  return v;
}

__device__ __forceinline__ uint4 lds_u128(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.b32 {%0,%1,%2,%3}, [%4];" : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}

// fp32 accumulation of binary16 products (sm_100 mixed-precision FMA): the
// product of two binary16 values is exact in fp32, so each term is added to
// the fp32 accumulator with a single fp32 rounding.  fma_lo uses the low
// halves of a and b, fma_hi the high halves.
__device__ __forceinline__ float fma_lo(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{ .reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1; mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %3; }"
      : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

__device__ __forceinline__ float fma_hi(uint32_t a, uint32_t b, float c) {
  float d;
  asm("{ .reg .b16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1; mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a1, b1, %3; }"
      : "=f"(d) : "r"(a), "r"(b), "f"(c));
  return d;
}

// Shared-memory byte address of the table entry of the code pair at bit BIT of
// a block (20 words): ((pair << 7) + lane_base), the pair field moved to bit 7
// with one shift (or funnel shift) and masked.
template <int BIT>
__device__ __forceinline__ uint32_t pair_addr(const uint4 (&cw)[5], uint32_t lane_base) {
  constexpr int wi = BIT >> 5, sh = BIT & 31;
  const uint32_t lo = word_of(cw, wi);
  uint32_t t;
  if constexpr (sh > 22) {
    t = __funnelshift_r(lo, word_of(cw, wi + 1), sh - 7);
  } else if constexpr (sh >= 7) {
    t = lo >> (sh - 7);
  } else {
    t = lo << (7 - sh);
  }
  return (t & (0x3ffu << 7)) + lane_base;
}

// Table entries (binary16 centroid pairs) of the 8 code pairs of round R8.
template <int R8>
__device__ __forceinline__ void round_entries(const uint4 (&cw)[5], uint32_t lane_base, uint32_t (&ent)[8]) {
  ent[0] = lds_u32(pair_addr<80 * R8 + 0>(cw, lane_base));
  ent[1] = lds_u32(pair_addr<80 * R8 + 10>(cw, lane_base));
  ent[2] = lds_u32(pair_addr<80 * R8 + 20>(cw, lane_base));
  ent[3] = lds_u32(pair_addr<80 * R8 + 30>(cw, lane_base));
  ent[4] = lds_u32(pair_addr<80 * R8 + 40>(cw, lane_base));
  ent[5] = lds_u32(pair_addr<80 * R8 + 50>(cw, lane_base));
  ent[6] = lds_u32(pair_addr<80 * R8 + 60>(cw, lane_base));
  ent[7] = lds_u32(pair_addr<80 * R8 + 70>(cw, lane_base));
}

// sum over 8 pairs of c-pair . x-pair, every binary16 product added to an
// fp32 accumulator (four accumulators: pair parity x half).
__device__ __forceinline__ float round_dot(const uint32_t (&ent)[8], uint32_t x0, uint32_t x1, uint32_t x2,
                                           uint32_t x3, uint32_t x4, uint32_t x5, uint32_t x6, uint32_t x7) {
  const uint32_t x[8] = {x0, x1, x2, x3, x4, x5, x6, x7};
  float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    a[2 * (p & 1)] = fma_lo(ent[p], x[p], a[2 * (p & 1)]);
    a[2 * (p & 1) + 1] = fma_hi(ent[p], x[p], a[2 * (p & 1) + 1]);
  }
  return (a[0] + a[1]) + (a[2] + a[3]);
}

// Dot products of one (row, block) of codes with MT rotated activation blocks
// in shared memory (xb_addr: shared address of token 0's block, tok_bytes per token).
template <int MT>
__device__ __forceinline__ void block_dot(const uint4 (&cw)[5], uint32_t lane_base, uint32_t xb_addr, int tok_bytes,
                                          float (&acc)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
#define HLWQ_ROUND(R8)                                                                                   \
  {                                                                                                      \
    uint32_t ent[8];                                                                                     \
    round_entries<R8>(cw, lane_base, ent);                                                               \
    _Pragma("unroll") for (int m = 0; m < MT; ++m) {                                                     \
      const uint4 xa = lds_u128(xb_addr + m * tok_bytes + 32 * (R8));                                    \
      const uint4 xc = lds_u128(xb_addr + m * tok_bytes + 32 * (R8) + 16);                               \
      acc[m] += round_dot(ent, xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w);                         \
    }                                                                                                    \
  }
  HLWQ_ROUND(0) HLWQ_ROUND(1) HLWQ_ROUND(2) HLWQ_ROUND(3) HLWQ_ROUND(4) HLWQ_ROUND(5) HLWQ_ROUND(6) HLWQ_ROUND(7)
#undef HLWQ_ROUND
}

// Single-token dot product with the rotated activation block held in registers
// (64 half2 words, xr[p] = (x[2p], x[2p+1])).
__device__ __forceinline__ float block_dot_reg(const uint4 (&cw)[5], uint32_t lane_base, const uint32_t (&xr)[64]) {
  float acc = 0.0f;
#define HLWQ_ROUND1(R8)                                                                                  \
  {                                                                                                      \
    uint32_t ent[8];                                                                                     \
    round_entries<R8>(cw, lane_base, ent);                                                               \
    acc += round_dot(ent, xr[8 * (R8)], xr[8 * (R8) + 1], xr[8 * (R8) + 2], xr[8 * (R8) + 3],           \
                     xr[8 * (R8) + 4], xr[8 * (R8) + 5], xr[8 * (R8) + 6], xr[8 * (R8) + 7]);           \
  }
  HLWQ_ROUND1(0) HLWQ_ROUND1(1) HLWQ_ROUND1(2) HLWQ_ROUND1(3)
  HLWQ_ROUND1(4) HLWQ_ROUND1(5) HLWQ_ROUND1(6) HLWQ_ROUND1(7)
#undef HLWQ_ROUND1
  return acc;
}

__device__ __forceinline__ uint32_t word10(const uint2 (&c)[5], int i) {
  const uint2 u = c[i >> 1];
  return (i & 1) ? u.y : u.x;
}

// Address of the table entry of pair p (0..31) of a half block (10 words).
template <int P>
__device__ __forceinline__ uint32_t half_pair_addr(const uint2 (&cw)[5], uint32_t lane_base) {
  constexpr int bit = 10 * P, wi = bit >> 5, sh = bit & 31;
  const uint32_t lo = word10(cw, wi);
  uint32_t t;
  if constexpr (sh > 22) {
    t = __funnelshift_r(lo, word10(cw, wi + 1), sh - 7);
  } else if constexpr (sh >= 7) {
    t = lo >> (sh - 7);
  } else {
    t = lo << (7 - sh);
  }
  return (t & (0x3ffu << 7)) + lane_base;
}

// 8 pairs, every binary16 product added to the fp32 accumulators a[4]
// (pair parity x half).
template <int P0>
__device__ __forceinline__ void half_round(const uint2 (&cw)[5], uint32_t lane_base, const uint32_t (&xr)[32],
                                           float (&a)[4]) {
  uint32_t e[8];
  e[0] = lds_u32(half_pair_addr<P0 + 0>(cw, lane_base));
  e[1] = lds_u32(half_pair_addr<P0 + 1>(cw, lane_base));
  e[2] = lds_u32(half_pair_addr<P0 + 2>(cw, lane_base));
  e[3] = lds_u32(half_pair_addr<P0 + 3>(cw, lane_base));
  e[4] = lds_u32(half_pair_addr<P0 + 4>(cw, lane_base));
  e[5] = lds_u32(half_pair_addr<P0 + 5>(cw, lane_base));
  e[6] = lds_u32(half_pair_addr<P0 + 6>(cw, lane_base));
  e[7] = lds_u32(half_pair_addr<P0 + 7>(cw, lane_base));
#pragma unroll
  for (int p = 0; p < 8; ++p) {
    a[2 * (p & 1)] = fma_lo(e[p], xr[P0 + p], a[2 * (p & 1)]);
    a[2 * (p & 1) + 1] = fma_hi(e[p], xr[P0 + p], a[2 * (p & 1) + 1]);
  }
}

// Single-token dot product of a half block (64 codes) with 64 rotated
// activation values held in registers (xr[p] = (x[2p], x[2p+1])).
__device__ __forceinline__ float half_dot_reg(const uint2 (&cw)[5], uint32_t lane_base, const uint32_t (&xr)[32]) {
  float a[4] = {0.0f, 0.0f, 0.0f, 0.0f};
  half_round<0>(cw, lane_base, xr, a);
  half_round<8>(cw, lane_base, xr, a);
  half_round<16>(cw, lane_base, xr, a);
  half_round<24>(cw, lane_base, xr, a);
  return (a[0] + a[1]) + (a[2] + a[3]);
}

// Processes all items of a CTA's virtual-row range.  rowfn(vrow) returns the
// matrix row (index into packed/norms) of a virtual row.  Each warp keeps a
// ring of kDepth items' codes in registers; prefetch() issues the first
// kDepth loads (the caller can then build tables while they are in flight) and
// run() consumes the items, refilling the ring.  Results go to
// slots[m][vrow][chunk] with every scale applied.
template <int C, int MT, typename RowFn, int kDepth_ = 3>
struct Engine {
  static constexpr int G = 32 / C;
  static constexpr int kDepth = kDepth_;
  uint4 cw[kDepth][5];
  float sc[kDepth];
  bool ok[kDepth];
  int nb, nvrows, nch, nitems;
  const uint8_t* packed;
  const uint16_t* norms;
  RowFn rowfn;

  __device__ __forceinline__ Engine(const uint8_t* p, const uint16_t* n, int nb_, int nvrows_, RowFn f)
      : nb(nb_), nvrows(nvrows_), packed(p), norms(n), rowfn(f) {
    nch = (nb + C - 1) / C;
    nitems = ((nvrows + G - 1) / G) * nch;
  }

  __device__ __forceinline__ void fetch(int it, int d) {
    const int lane = threadIdx.x & 31;
    const int r = lane / C, s = lane % C;
    ok[d] = false;
    sc[d] = 0.0f;
    if (it >= nitems) return;
    const int g = it / nch, ch = it - g * nch;
    const int vrow = g * G + r, b = ch * C + s;
    if (vrow < nvrows && b < nb) {
      const int64_t F = rowfn(vrow) * static_cast<int64_t>(nb) + b;
      const uint4* src = reinterpret_cast<const uint4*>(packed + F * kBlockBytes);
#pragma unroll
      for (int q = 0; q < 5; ++q) cw[d][q] = ldg_stream(src + q);
      sc[d] = half_bits_to_float(__ldg(norms + F)) * (1.0f / 128.0f);
      ok[d] = true;
    }
  }

  __device__ __forceinline__ void prefetch() {
    const int warp = threadIdx.x >> 5;
#pragma unroll
    for (int d = 0; d < kDepth; ++d) fetch(warp + d * kEngineWarps, d);
  }

  __device__ __forceinline__ void consume(int it, int d, uint32_t lane_base, uint32_t xs_addr,
                                          const float* __restrict__ xinv, float* __restrict__ slots) {
    const int lane = threadIdx.x & 31;
    const int r = lane / C, s = lane % C;
    const int g = it / nch, ch = it - g * nch;
    const int b = ch * C + s;
    float acc[MT];
    if (ok[d]) {
      block_dot<MT>(cw[d], lane_base, xs_addr + b * (kXsStride * 2), nb * kXsStride * 2, acc);
#pragma unroll
      for (int m = 0; m < MT; ++m) acc[m] *= sc[d] * xinv[m * nb + b];
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
  }

  __device__ __forceinline__ void run(const uint32_t* __restrict__ tab, const uint16_t* __restrict__ xs,
                                      const float* __restrict__ xinv, float* __restrict__ slots) {
    const int warp = threadIdx.x >> 5;
    const uint32_t lane_base = static_cast<uint32_t>(__cvta_generic_to_shared(tab)) + 4u * (threadIdx.x & 31);
    const uint32_t xs_addr = static_cast<uint32_t>(__cvta_generic_to_shared(xs));
    for (int base = warp; base < nitems; base += kDepth * kEngineWarps) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int it = base + d * kEngineWarps;
        if (it < nitems) {
          consume(it, d, lane_base, xs_addr, xinv, slots);
          fetch(it + kDepth * kEngineWarps, d);
        }
      }
    }
  }
};

template <int C, int MT, int kDepth = 3, typename RowFn>
__device__ __forceinline__ Engine<C, MT, RowFn, kDepth> make_engine(const uint8_t* p, const uint16_t* n, int nb,
                                                                    int nvrows, RowFn f) {
  return Engine<C, MT, RowFn, kDepth>(p, n, nb, nvrows, f);
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
