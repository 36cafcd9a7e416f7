#pragma once
// TQ3 weights (the scalar case of HIGGS) on sm_100a: quantizer, dequantizer
// and the decode GEMV on the 3-bit codes ("Qwen3.6-35B-A3B-TQ3-native", "What
// TQ3 actually does" and "Files").
//
// Per row and group g of 128 inputs (tail zero-padded), with the sign vectors
// s1, s2 (+-1, one pair for every group) and the 8 fp32 Lloyd-Max centroids c:
//   n      = ||g||_2
//   y      = s2 * (H128 (s1 * g)) / n                (y = 0 if n = 0)
//   code_j = number of decision midpoints below y_j  (nearest centroid, ties low)
//   gamma  = n / sqrt(||c[code]||^2 / 128)           (0 for a zero group), fp32
//   packed : code j at bits [3j, 3j + 3) of the group's 48 bytes, LSB first
// Dequantized group: w_hat = gamma * s1 * (H128 (s2 * c[code])) / 128, so that
// ||w_hat|| = n.
//
// Quantizer: four lanes per group, 32 values each, all in fp64.  The +-1 sums
// of bf16 values are exact in fp64, and n, y and the midpoint comparisons are
// correctly rounded fp64 operations, so the codes are those of the fp64
// definition.  ||c[code]||^2 is formed from the per-level code counts as
// sum_l m_l * c_l^2, levels in ascending order (m_l * c_l^2 rounded, then
// added), so gamma is bit-for-bit that of any evaluation in that order.
//
// GEMV, y[o] = sum_b gamma[o][b] / 128 * sum_j c[k_obj] xt_b[j] with
// xt_b = s2 * (H128 (s1 * x_b)): the activation is rotated once and the codes
// are dotted with it in the rotated domain.  The inputs are cut into slices of
// 1024 (8 groups); a lane owns 32 positions of a slice (a quarter group), so
// its share of every row is 96 bits of codes.  For its slice a CTA tabulates,
// per lane and per pair of the lane's positions, c[a] xt[2p] + c[b] xt[2p+1]
// for all 64 code pairs (a, b): 16 pairs x 64 x 32 lanes x 4 bytes = 128 KiB of
// shared memory, laid out [pair][a + 8b][lane] so that every lookup of a warp
// hits 32 distinct banks.  A row's share then costs 16 table lookups and adds
// per lane.  Eight rows are reduced over the warp at a time by a transposed
// butterfly (9 shuffles).  The slices of a row range are handled by the CTAs
// of one thread-block cluster (one CTA per slice, up to 8; more slices are
// taken in turn); each CTA keeps its slice sums in shared memory and, after a
// cluster barrier, every CTA adds up a part of the rows over the cluster's
// CTAs in rank order through distributed shared memory and writes y.

#include <utility>

#include "hlwq_common.cuh"

namespace hlwq {

namespace {

constexpr int kT3Levels = 8;
constexpr int kT3GroupBytes = 48;
constexpr int kT3QThreads = 256;

__device__ __forceinline__ void t3_check_codebook(const float* cb) {
  if (threadIdx.x + 1 < kT3Levels) {
    const float a = __ldg(cb + threadIdx.x), b = __ldg(cb + threadIdx.x + 1);
    if (!(a < b) || !isfinite(a) || !isfinite(b)) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
}

__device__ __forceinline__ double quad_sum_f64(double x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  return x + __shfl_xor_sync(0xffffffffu, x, 2);
}

// Bit e set where entry base + e of a sign vector is negative (-1); every
// other value counts as +1.
__device__ __forceinline__ uint32_t t3_sign_mask(const int8_t* __restrict__ s, int base) {
  uint32_t m = 0u;
#pragma unroll
  for (int e = 0; e < 32; ++e) m |= (__ldg(s + base + e) < 0 ? 1u : 0u) << e;
  return m;
}

// 32 values of a row starting at column col0 (bf16 -> fp64, zero beyond `in`).
__device__ __forceinline__ void t3_load_quarter(const uint16_t* __restrict__ row, int col0, int in, bool vec,
                                                bool active, double (&v)[32]) {
  const int qlen = active ? max(0, min(32, in - col0)) : 0;
  if (vec) {
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      uint4 u = make_uint4(0u, 0u, 0u, 0u);
      if (8 * c < qlen) u = __ldg(reinterpret_cast<const uint4*>(row + col0) + c);
      const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        v[8 * c + 2 * k] = static_cast<double>(__uint_as_float(wd[k] << 16));
        v[8 * c + 2 * k + 1] = static_cast<double>(__uint_as_float(wd[k] & 0xffff0000u));
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      v[e] = e < qlen ? static_cast<double>(__uint_as_float(static_cast<uint32_t>(__ldg(row + col0 + e)) << 16)) : 0.0;
  }
}

__global__ void __launch_bounds__(kT3QThreads)
tq3_quantize_kernel(const uint16_t* __restrict__ W, int64_t rows, int in, int nb, const int8_t* __restrict__ signs,
                    const float* __restrict__ codebook, uint8_t* __restrict__ packed, float* __restrict__ norms,
                    int vec) {
  __shared__ double mid[kT3Levels - 1];
  __shared__ double csq[kT3Levels];
  t3_check_codebook(codebook);
  if (threadIdx.x < kT3Levels - 1)
    mid[threadIdx.x] = 0.5 * (static_cast<double>(__ldg(codebook + threadIdx.x)) +
                              static_cast<double>(__ldg(codebook + threadIdx.x + 1)));
  if (threadIdx.x < kT3Levels) {
    const double c = static_cast<double>(__ldg(codebook + threadIdx.x));
    csq[threadIdx.x] = c * c;  // exact: a 24-bit significand squared
  }
  __syncthreads();
  const int lane = threadIdx.x & 31, q = lane & 3;
  const uint32_t m1 = t3_sign_mask(signs, 32 * q), m2 = t3_sign_mask(signs, kBlock + 32 * q);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kT3QThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kT3QThreads / 32);
  const int64_t ngroups = rows * nb;
  for (int64_t first = warp * 8; first < ngroups; first += nwarps * 8) {
    const int64_t G = first + (lane >> 2);
    const bool active = G < ngroups;
    const int64_t o = active ? G / nb : 0;
    const int b = active ? static_cast<int>(G - o * nb) : 0;
    double v[32];
    t3_load_quarter(W + o * in, kBlock * b + 32 * q, in, vec != 0, active, v);
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fma(v[e], v[e], ss);
    ss = quad_sum_f64(ss);
    const double nrm = sqrt(ss);
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = (m1 >> e) & 1u ? -v[e] : v[e];
    kv_stage<double, 1>(v);
    kv_stage<double, 2>(v);
    kv_stage<double, 4>(v);
    kv_stage<double, 8>(v);
    kv_stage<double, 16>(v);
    kv_stage_x<double, 1>(v, lane);
    kv_stage_x<double, 2>(v, lane);
    uint32_t w[3] = {0u, 0u, 0u};
    uint64_t counts = 0ull;  // 8 bits per level
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const double y = nrm > 0.0 ? ((m2 >> e) & 1u ? -v[e] : v[e]) / nrm : 0.0;
      uint32_t code = 0u;
#pragma unroll
      for (int k = 0; k < kT3Levels - 1; ++k) code += y > mid[k] ? 1u : 0u;
      counts += 1ull << (8 * code);
      const int bit = 3 * e, k = bit >> 5, sh = bit & 31;
      w[k] |= code << sh;
      if (sh > 29) w[k + 1] |= code >> (32 - sh);
    }
    counts += __shfl_xor_sync(0xffffffffu, counts, 1);
    counts += __shfl_xor_sync(0xffffffffu, counts, 2);
    double r2 = 0.0;
#pragma unroll
    for (int l = 0; l < kT3Levels; ++l)
      r2 = __dadd_rn(r2, __dmul_rn(static_cast<double>((counts >> (8 * l)) & 0xffull), csq[l]));
    const double gamma = nrm > 0.0 ? nrm / sqrt(r2 * (1.0 / kBlock)) : 0.0;
    if (active) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(packed + G * kT3GroupBytes + 12 * q);
      dst[0] = w[0];
      dst[1] = w[1];
      dst[2] = w[2];
      if (q == 0) norms[G] = __double2float_rn(gamma);
    }
  }
}

template <bool kOutBf16, bool kVec>
__global__ void __launch_bounds__(kT3QThreads)
tq3_dequantize_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ norms,
                      const int8_t* __restrict__ signs, const float* __restrict__ codebook, int64_t rows, int in,
                      int nb, void* __restrict__ out) {
  __shared__ float cb[kT3Levels];
  t3_check_codebook(codebook);
  if (threadIdx.x < kT3Levels) cb[threadIdx.x] = __ldg(codebook + threadIdx.x);
  __syncthreads();
  const int lane = threadIdx.x & 31, q = lane & 3;
  const uint32_t m1 = t3_sign_mask(signs, 32 * q), m2 = t3_sign_mask(signs, kBlock + 32 * q);
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kT3QThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kT3QThreads / 32);
  const int64_t ngroups = rows * nb;
  for (int64_t first = warp * 8; first < ngroups; first += nwarps * 8) {
    const int64_t G = first + (lane >> 2);
    const bool active = G < ngroups;
    uint32_t w[3] = {0u, 0u, 0u};
    float scale = 0.0f;
    int64_t o = 0;
    int b = 0;
    if (active) {
      o = G / nb;
      b = static_cast<int>(G - o * nb);
      const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + G * kT3GroupBytes + 12 * q);
      w[0] = __ldg(src);
      w[1] = __ldg(src + 1);
      w[2] = __ldg(src + 2);
      scale = __ldg(norms + G) * (1.0f / kBlock);
    }
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const float t = cb[kv_code(w, e)];
      v[e] = (m2 >> e) & 1u ? -t : t;
    }
    fwht_4lanes(v, lane);
    const int qlen = active ? max(0, min(32, in - kBlock * b - 32 * q)) : 0;
    if (qlen == 0) continue;
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] *= (m1 >> e) & 1u ? -scale : scale;
    const int64_t off = o * static_cast<int64_t>(in) + static_cast<int64_t>(kBlock) * b + 32 * q;
    if constexpr (!kOutBf16) {
      float* dst = static_cast<float*>(out) + off;
      if constexpr (kVec) {
#pragma unroll
        for (int c = 0; c < 8; ++c)
          if (4 * c < qlen) reinterpret_cast<float4*>(dst)[c] = make_float4(v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3]);
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < qlen) dst[e] = v[e];
      }
    } else {
      uint16_t* dst = static_cast<uint16_t*>(out) + off;
      if constexpr (kVec) {
#pragma unroll
        for (int c = 0; c < 4; ++c)
          if (8 * c < qlen) {
            uint4 u;
            u.x = float_to_bf16_bits(v[8 * c]) | (float_to_bf16_bits(v[8 * c + 1]) << 16);
            u.y = float_to_bf16_bits(v[8 * c + 2]) | (float_to_bf16_bits(v[8 * c + 3]) << 16);
            u.z = float_to_bf16_bits(v[8 * c + 4]) | (float_to_bf16_bits(v[8 * c + 5]) << 16);
            u.w = float_to_bf16_bits(v[8 * c + 6]) | (float_to_bf16_bits(v[8 * c + 7]) << 16);
            reinterpret_cast<uint4*>(dst)[c] = u;
          }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e)
          if (e < qlen) dst[e] = static_cast<uint16_t>(float_to_bf16_bits(v[e]));
      }
    }
  }
}

// ---------------------------------------------------------------- GEMV
constexpr int kT3GThreads = 512;
constexpr int kT3GWarps = kT3GThreads / 32;
constexpr int kT3SliceGroups = 8;                                // groups per slice
constexpr int kT3Slice = kT3SliceGroups * kBlock;                // 1024 inputs
constexpr int kT3TableBytes = 16 * 64 * 32 * 4;                  // [pair][a + 8b][lane] fp32
constexpr int kT3ChunkRows = 4096;                               // slice sums kept per pass
constexpr int kT3SmemBytes = 8192 + kT3TableBytes + kT3Slice * 4 + kT3ChunkRows * 4;  // + alignment slack
constexpr int kT3MaxCluster = 8;

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ uint32_t cluster_size() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// fp32 at the same shared-memory offset in the CTA of cluster rank `rank`.
__device__ __forceinline__ float ld_cluster_f32(const float* local, uint32_t rank) {
  const uint32_t a = static_cast<uint32_t>(__cvta_generic_to_shared(local));
  uint32_t ra;
  float v;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(ra) : "r"(a), "r"(rank));
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(ra) : "memory");
  return v;
}

// Table lookup of pair P of a lane's 96-bit code string (w0, w1, w2): the
// 6-bit field at bits [6P, 6P + 6) moved to bit 7 (index times 128 bytes) and
// or'ed into `lb` (the 8 KiB-aligned table address with the lane's 4-byte
// column) -- one shift and one lop3 -- then read at the immediate offset
// P * 8192 of the pair's table block.
template <int P>
__device__ __forceinline__ float t3_lookup(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t lb) {
  constexpr int bit = 6 * P, k = bit >> 5, sh = bit & 31;
  const uint32_t lo = k == 0 ? w0 : (k == 1 ? w1 : w2);
  float t;
  if constexpr (sh > 26) {
    // the field crosses into the next word: funnel shift it to bit 7
    const uint32_t hi = k == 0 ? w1 : w2;
    asm volatile(
        "{ .reg .b32 a;\n\t"
        "shf.r.clamp.b32 a, %1, %2, %3;\n\t"
        "lop3.b32 a, a, 0x1f80, %4, 0xea;\n\t"
        "ld.shared.f32 %0, [a+%5]; }"
        : "=f"(t)
        : "r"(lo), "r"(hi), "n"(sh - 7), "r"(lb), "n"(P * 8192));
  } else if constexpr (sh >= 7) {
    asm volatile(
        "{ .reg .b32 a;\n\t"
        "shr.b32 a, %1, %2;\n\t"
        "lop3.b32 a, a, 0x1f80, %3, 0xea;\n\t"
        "ld.shared.f32 %0, [a+%4]; }"
        : "=f"(t)
        : "r"(lo), "n"(sh - 7), "r"(lb), "n"(P * 8192));
  } else {
    asm volatile(
        "{ .reg .b32 a;\n\t"
        "shl.b32 a, %1, %2;\n\t"
        "lop3.b32 a, a, 0x1f80, %3, 0xea;\n\t"
        "ld.shared.f32 %0, [a+%4]; }"
        : "=f"(t)
        : "r"(lo), "n"(7 - sh), "r"(lb), "n"(P * 8192));
  }
  return t;
}

template <int... P>
__device__ __forceinline__ float t3_row_sum(uint32_t w0, uint32_t w1, uint32_t w2, uint32_t lb,
                                            std::integer_sequence<int, P...>) {
  float t[sizeof...(P)] = {t3_lookup<P>(w0, w1, w2, lb)...};
  float a0 = 0.0f, a1 = 0.0f, a2 = 0.0f, a3 = 0.0f;
#pragma unroll
  for (int i = 0; i < static_cast<int>(sizeof...(P)); i += 4) {
    a0 += t[i];
    a1 += t[i + 1];
    a2 += t[i + 2];
    a3 += t[i + 3];
  }
  return (a0 + a1) + (a2 + a3);
}

// Eight values per lane -> the sum over the warp of value i, held by the lanes
// whose bits 4..2 equal i (lane >> 2 == i); 9 shuffles.
__device__ __forceinline__ float t3_reduce8(float (&v)[8], int lane) {
  const bool u16 = (lane & 16) != 0, u8 = (lane & 8) != 0, u4 = (lane & 4) != 0;
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const float send = u16 ? v[i] : v[i + 4], keep = u16 ? v[i + 4] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 16);
  }
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const float send = u8 ? v[i] : v[i + 2], keep = u8 ? v[i + 2] : v[i];
    v[i] = keep + __shfl_xor_sync(0xffffffffu, send, 8);
  }
  const float send = u4 ? v[0] : v[1], keep = u4 ? v[1] : v[0];
  float r = keep + __shfl_xor_sync(0xffffffffu, send, 4);
  r += __shfl_xor_sync(0xffffffffu, r, 1);
  return r + __shfl_xor_sync(0xffffffffu, r, 2);
}

// Codes and norms of the eight rows c0 + 8g .. c0 + 8g + 7 for the lane's
// group gb (zeros where a row or the group does not exist).
__device__ __forceinline__ void t3_load_rows(const uint8_t* __restrict__ packed, const float* __restrict__ norms,
                                             int64_t c0, int g, int nrows, int nb, int gb, bool gvalid, int q,
                                             uint32_t (&w)[8][3], float (&gm)[8]) {
  const int64_t first = c0 + 8 * g;
  const uint8_t* pc = packed + (first * nb + gb) * kT3GroupBytes + 12 * q;
  const float* pn = norms + first * nb + gb;
  const int64_t rs = static_cast<int64_t>(nb) * kT3GroupBytes;
  if (gvalid && 8 * g + 8 <= nrows) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(pc + i * rs);
      w[i][0] = __ldg(src);
      w[i][1] = __ldg(src + 1);
      w[i][2] = __ldg(src + 2);
      gm[i] = __ldg(pn + static_cast<int64_t>(i) * nb);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      w[i][0] = w[i][1] = w[i][2] = 0u;
      gm[i] = 0.0f;
      if (gvalid && 8 * g + i < nrows) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(pc + i * rs);
        w[i][0] = __ldg(src);
        w[i][1] = __ldg(src + 1);
        w[i][2] = __ldg(src + 2);
        gm[i] = __ldg(pn + static_cast<int64_t>(i) * nb);
      }
    }
  }
}

// Sums of eight rows' shares (rows i0 .. i0 + 7 of the pass) into acc.
__device__ __forceinline__ void t3_rows_step(const uint32_t (&w)[8][3], const float (&gm)[8], uint32_t lb, int lane,
                                             int q, int i0, int nrows, float* acc) {
  float v[8];
#pragma unroll
  for (int i = 0; i < 8; ++i)
    v[i] = t3_row_sum(w[i][0], w[i][1], w[i][2], lb, std::make_integer_sequence<int, 16>{}) * gm[i];
  const float r = t3_reduce8(v, lane);
  const int i = i0 + (lane >> 2);
  if (q == 0 && i < nrows) acc[i] += r;
}

__global__ void __launch_bounds__(kT3GThreads, 1)
tq3_gemv_kernel(const uint8_t* __restrict__ packed, const float* __restrict__ norms,
                const int8_t* __restrict__ signs, const float* __restrict__ codebook, int64_t O, int in, int nb,
                int nslices, int64_t rows_per_cluster, const uint16_t* __restrict__ x, void* __restrict__ y,
                int out_bf16, int xvec) {
  extern __shared__ __align__(16) unsigned char t3s[];
  // the table starts on an 8 KiB boundary, so a lookup address is the
  // table's address or'ed with the lane column and the code-pair index
  const uint32_t raw = static_cast<uint32_t>(__cvta_generic_to_shared(t3s));
  const uint32_t pad = (8192u - (raw & 8191u)) & 8191u;
  unsigned char* tbl = t3s + pad;
  float* xr = reinterpret_cast<float*>(tbl + kT3TableBytes);
  float* acc = xr + kT3Slice;
  const uint32_t C = cluster_size(), rank = cluster_rank();
  const int64_t cid = blockIdx.x / C;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, q = lane & 3;
  const uint32_t lb = (raw + pad) | (static_cast<uint32_t>(lane) * 4u);
  t3_check_codebook(codebook);
  float c[kT3Levels];
#pragma unroll
  for (int k = 0; k < kT3Levels; ++k) c[k] = __ldg(codebook + k);
  const int64_t r0 = cid * rows_per_cluster;
  const int64_t r1 = min(O, r0 + rows_per_cluster);
  for (int64_t c0 = r0; c0 < r1; c0 += kT3ChunkRows) {
    const int nrows = static_cast<int>(min(static_cast<int64_t>(kT3ChunkRows), r1 - c0));
    for (int i = threadIdx.x; i < nrows; i += kT3GThreads) acc[i] = 0.0f;
    for (int s = static_cast<int>(rank); s < nslices; s += static_cast<int>(C)) {
      const int gb = s * kT3SliceGroups + (lane >> 2);
      const bool gvalid = gb < nb;
      // the first rows' codes are requested before the table is built
      uint32_t wc[8][3];
      float gc[8];
      t3_load_rows(packed, norms, c0, warp, nrows, nb, gb, gvalid, q, wc, gc);
      __syncthreads();  // readers of the previous table are done; acc is zeroed
      if (warp == 0) {
        // xt for the slice: lane holds positions 32 lane .. 32 lane + 31
        float v[32];
        const int col0 = kBlock * gb + 32 * q;
        const int qlen = gvalid ? max(0, min(32, in - col0)) : 0;
        if (xvec) {
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            uint4 u = make_uint4(0u, 0u, 0u, 0u);
            if (8 * k < qlen) u = __ldg(reinterpret_cast<const uint4*>(x + col0) + k);
            const uint32_t wd[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              v[8 * k + 2 * j] = bf16x2_lo(wd[j]);
              v[8 * k + 2 * j + 1] = bf16x2_hi(wd[j]);
            }
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) v[e] = e < qlen ? bf16_bits_to_float(__ldg(x + col0 + e)) : 0.0f;
        }
        const uint32_t m1 = t3_sign_mask(signs, 32 * q), m2 = t3_sign_mask(signs, kBlock + 32 * q);
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = (m1 >> e) & 1u ? -v[e] : v[e];
        fwht_4lanes(v, lane);
        float4* dst = reinterpret_cast<float4*>(xr + 32 * lane);
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float4 f;
          f.x = (m2 >> (4 * k)) & 1u ? -v[4 * k] : v[4 * k];
          f.y = (m2 >> (4 * k + 1)) & 1u ? -v[4 * k + 1] : v[4 * k + 1];
          f.z = (m2 >> (4 * k + 2)) & 1u ? -v[4 * k + 2] : v[4 * k + 2];
          f.w = (m2 >> (4 * k + 3)) & 1u ? -v[4 * k + 3] : v[4 * k + 3];
          dst[k] = f;
        }
      }
      __syncthreads();
      {
        // table block of pair p = warp: entry [a + 8b][lane] = c[a] xt[2p] + c[b] xt[2p + 1]
        const float2 xx = *reinterpret_cast<const float2*>(xr + 32 * lane + 2 * warp);
        float* tb = reinterpret_cast<float*>(tbl + warp * 8192) + lane;
#pragma unroll
        for (int b = 0; b < kT3Levels; ++b) {
          const float hb = c[b] * xx.y;
#pragma unroll
          for (int a = 0; a < kT3Levels; ++a) tb[(a + 8 * b) * 32] = fmaf(c[a], xx.x, hb);
        }
      }
      __syncthreads();
      // two register sets in turn: the next group's codes are in flight while
      // the current group is summed
      uint32_t wn[8][3];
      float gn[8];
      for (int g = warp; 8 * g < nrows; g += 2 * kT3GWarps) {
        t3_load_rows(packed, norms, c0, g + kT3GWarps, nrows, nb, gb, gvalid, q, wn, gn);
        t3_rows_step(wc, gc, lb, lane, q, 8 * g, nrows, acc);
        if (8 * (g + kT3GWarps) >= nrows) break;
        t3_load_rows(packed, norms, c0, g + 2 * kT3GWarps, nrows, nb, gb, gvalid, q, wc, gc);
        t3_rows_step(wn, gn, lb, lane, q, 8 * (g + kT3GWarps), nrows, acc);
      }
    }
    cluster_sync_all();  // every CTA of the cluster has its slice sums of the chunk
    const int per = (nrows + static_cast<int>(C) - 1) / static_cast<int>(C);
    const int i0 = static_cast<int>(rank) * per, i1 = min(nrows, i0 + per);
    for (int i = i0 + threadIdx.x; i < i1; i += kT3GThreads) {
      float sum = 0.0f;
      for (uint32_t k = 0; k < C; ++k) sum += ld_cluster_f32(acc + i, k);
      sum *= 1.0f / kBlock;
      if (out_bf16) static_cast<uint16_t*>(y)[c0 + i] = static_cast<uint16_t>(float_to_bf16_bits(sum));
      else static_cast<float*>(y)[c0 + i] = sum;
    }
    cluster_sync_all();  // no CTA re-zeroes or leaves while another reads its sums
  }
}

}  // namespace

int launch_tq3_quantize(const uint16_t* W, int64_t rows, int in, const int8_t* signs, const float* codebook,
                        uint8_t* packed, float* norms, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int64_t ngroups = rows * nb;
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(ngroups, kT3QThreads / 4)));
  const int vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) && (in % 8 == 0);
  tq3_quantize_kernel<<<grid, kT3QThreads, 0, stream>>>(W, rows, in, nb, signs, codebook, packed, norms, vec);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_tq3_dequantize(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                          int64_t rows, int in, void* out, bool bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int64_t ngroups = rows * nb;
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(ngroups, kT3QThreads / 4)));
  const bool vec = (reinterpret_cast<uintptr_t>(out) % 16 == 0) &&
                   ((static_cast<int64_t>(in) * (bf16 ? 2 : 4)) % 16 == 0);
  if (bf16) {
    if (vec) tq3_dequantize_kernel<true, true><<<grid, kT3QThreads, 0, stream>>>(packed, norms, signs, codebook, rows, in, nb, out);
    else tq3_dequantize_kernel<true, false><<<grid, kT3QThreads, 0, stream>>>(packed, norms, signs, codebook, rows, in, nb, out);
  } else {
    if (vec) tq3_dequantize_kernel<false, true><<<grid, kT3QThreads, 0, stream>>>(packed, norms, signs, codebook, rows, in, nb, out);
    else tq3_dequantize_kernel<false, false><<<grid, kT3QThreads, 0, stream>>>(packed, norms, signs, codebook, rows, in, nb, out);
  }
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_tq3_gemv(const uint8_t* packed, const float* norms, const int8_t* signs, const float* codebook,
                    int64_t O, int in, const uint16_t* x, void* y, bool out_bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int nslices = static_cast<int>(ceil_div(nb, kT3SliceGroups));
  const int C = std::min(nslices, kT3MaxCluster);
  static PerDeviceOnce attr;
  if (const int st = attr([&] {
        return cudaFuncSetAttribute(tq3_gemv_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kT3SmemBytes) == cudaSuccess;
      }))
    return st;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeClusterDimension;
  at[0].val.clusterDim.x = C;
  at[0].val.clusterDim.y = 1;
  at[0].val.clusterDim.z = 1;
  cfg.blockDim = dim3(kT3GThreads);
  cfg.dynamicSmemBytes = kT3SmemBytes;
  cfg.stream = stream;
  cfg.attrs = at;
  cfg.numAttrs = 1;
  // co-resident clusters of this size (cached per size and device)
  static int max_clusters[kT3MaxCluster + 1][64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  int& mc = max_clusters[C][dev & 63];
  if (mc == 0) {
    cfg.gridDim = dim3(C);
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, tq3_gemv_kernel, &cfg) != cudaSuccess || n <= 0) return HLWQ_ECUDA;
    mc = n;
  }
  const int64_t nclusters = std::max<int64_t>(1, std::min<int64_t>(mc, ceil_div(O, 8)));
  const int64_t rows_per_cluster = ceil_div(ceil_div(O, nclusters), 8) * 8;
  const int64_t used = ceil_div(O, rows_per_cluster);
  cfg.gridDim = dim3(static_cast<unsigned>(used * C));
  const int xvec = (reinterpret_cast<uintptr_t>(x) % 16 == 0) && (in % 8 == 0);
  if (cudaLaunchKernelEx(&cfg, tq3_gemv_kernel, packed, norms, signs, codebook, O, in, nb, nslices, rows_per_cluster,
                         x, y, static_cast<int>(out_bf16), xvec) != cudaSuccess)
    return HLWQ_ECUDA;
  return HLWQ_OK;
}

}  // namespace hlwq
