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
// scaled by a power of two per 128-block; products are formed with packed
// half2 FMAs in short chains (at most 4 products per chain, combined pairwise)
// and every 16 products are added to an fp32 accumulator.
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

__device__ __forceinline__ __half2 u2h(uint32_t v) { return *reinterpret_cast<const __half2*>(&v); }

// Table entries of the 8 code pairs of round r8 (pairs 8 r8 .. 8 r8 + 7).
template <int R8>
__device__ __forceinline__ void round_entries(const uint4 (&cw)[5], const uint32_t* __restrict__ tab_lane,
                                              uint32_t (&ent)[8]) {
#pragma unroll
  for (int t = 0; t < 8; ++t) {
    const int bit = 80 * R8 + 10 * t, wi = bit >> 5, sh = bit & 31;
    const uint32_t lo = word_of(cw, wi);
    const uint32_t hi = (wi + 1 < 20) ? word_of(cw, wi + 1) : 0u;
    const uint32_t v10 = (sh <= 22) ? ((lo >> sh) & 0x3ffu) : (__funnelshift_r(lo, hi, sh) & 0x3ffu);
    ent[t] = tab_lane[v10 << 5];
  }
}

// sum_t c-pair(ent[t]) . x-pair(x[t]) for 8 pairs: four half2 product chains of
// two pairs each, combined pairwise in half2 and finally in fp32 (the rotated
// activation is scaled so that |x| < 2^10, far from binary16 overflow).
__device__ __forceinline__ float round_dot(const uint32_t (&ent)[8], uint32_t x0, uint32_t x1, uint32_t x2,
                                           uint32_t x3, uint32_t x4, uint32_t x5, uint32_t x6, uint32_t x7) {
  __half2 h0 = __hmul2(u2h(ent[0]), u2h(x0));
  __half2 h1 = __hmul2(u2h(ent[1]), u2h(x1));
  __half2 h2 = __hmul2(u2h(ent[2]), u2h(x2));
  __half2 h3 = __hmul2(u2h(ent[3]), u2h(x3));
  h0 = __hfma2(u2h(ent[4]), u2h(x4), h0);
  h1 = __hfma2(u2h(ent[5]), u2h(x5), h1);
  h2 = __hfma2(u2h(ent[6]), u2h(x6), h2);
  h3 = __hfma2(u2h(ent[7]), u2h(x7), h3);
  const float2 f = __half22float2(__hadd2(__hadd2(h0, h1), __hadd2(h2, h3)));
  return f.x + f.y;
}

// Dot products of one (row, block) of codes with MT rotated activation blocks
// stored in shared memory (xb: block base of token 0, xs_tok_stride halves per token).
template <int MT>
__device__ __forceinline__ void block_dot(const uint4 (&cw)[5], const uint32_t* __restrict__ tab_lane,
                                          const uint16_t* __restrict__ xb, int xs_tok_stride, float (&acc)[MT]) {
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m] = 0.0f;
#define HLWQ_ROUND(R8)                                                                                   \
  {                                                                                                      \
    uint32_t ent[8];                                                                                     \
    round_entries<R8>(cw, tab_lane, ent);                                                                \
    _Pragma("unroll") for (int m = 0; m < MT; ++m) {                                                     \
      const uint4 xa = *reinterpret_cast<const uint4*>(xb + m * xs_tok_stride + 16 * (R8));             \
      const uint4 xc = *reinterpret_cast<const uint4*>(xb + m * xs_tok_stride + 16 * (R8) + 8);         \
      acc[m] += round_dot(ent, xa.x, xa.y, xa.z, xa.w, xc.x, xc.y, xc.z, xc.w);                         \
    }                                                                                                    \
  }
  HLWQ_ROUND(0) HLWQ_ROUND(1) HLWQ_ROUND(2) HLWQ_ROUND(3) HLWQ_ROUND(4) HLWQ_ROUND(5) HLWQ_ROUND(6) HLWQ_ROUND(7)
#undef HLWQ_ROUND
}

// Single-token dot product with the rotated activation block held in registers
// (64 half2 words, xr[p] = (x[2p], x[2p+1])).
__device__ __forceinline__ float block_dot_reg(const uint4 (&cw)[5], const uint32_t* __restrict__ tab_lane,
                                               const uint32_t (&xr)[64]) {
  float acc = 0.0f;
#define HLWQ_ROUND1(R8)                                                                                  \
  {                                                                                                      \
    uint32_t ent[8];                                                                                     \
    round_entries<R8>(cw, tab_lane, ent);                                                                \
    acc += round_dot(ent, xr[8 * (R8)], xr[8 * (R8) + 1], xr[8 * (R8) + 2], xr[8 * (R8) + 3],           \
                     xr[8 * (R8) + 4], xr[8 * (R8) + 5], xr[8 * (R8) + 6], xr[8 * (R8) + 7]);           \
  }
  HLWQ_ROUND1(0) HLWQ_ROUND1(1) HLWQ_ROUND1(2) HLWQ_ROUND1(3)
  HLWQ_ROUND1(4) HLWQ_ROUND1(5) HLWQ_ROUND1(6) HLWQ_ROUND1(7)
#undef HLWQ_ROUND1
  return acc;
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

  __device__ __forceinline__ void consume(int it, int d, const uint32_t* __restrict__ tab_lane,
                                          const uint16_t* __restrict__ xs, const float* __restrict__ xinv,
                                          float* __restrict__ slots) {
    const int lane = threadIdx.x & 31;
    const int r = lane / C, s = lane % C;
    const int g = it / nch, ch = it - g * nch;
    const int b = ch * C + s;
    float acc[MT];
    if (ok[d]) {
      block_dot<MT>(cw[d], tab_lane, xs + b * kXsStride, nb * kXsStride, acc);
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
    const uint32_t* tab_lane = tab + (threadIdx.x & 31);
    for (int base = warp; base < nitems; base += kDepth * kEngineWarps) {
#pragma unroll
      for (int d = 0; d < kDepth; ++d) {
        const int it = base + d * kEngineWarps;
        if (it < nitems) {
          consume(it, d, tab_lane, xs, xinv, slots);
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
