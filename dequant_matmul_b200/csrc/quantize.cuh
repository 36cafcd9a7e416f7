#pragma once
// HLWQ Q5 quantizer and dequantizer kernels (sm_100a).
//
// Quantizer ("Qwen3.6-35B-A3B -- HLWQ Q5" model card, Method steps [1]-[5]):
// one thread owns one 128-weight block; the block lives in 128 fp32 registers,
// so the Walsh-Hadamard rotation is seven in-register butterfly stages with no
// shuffles or shared-memory traffic.  Weights are read with 16-byte loads
// straight into registers (each warp covers 32 consecutive blocks, so a warp's
// loads cover a contiguous span of the weight matrix).
//
// Nearest-centroid assignment (step [4]) uses a 2048-entry bucket table in
// shared memory: y is mapped to a bucket of width 1/64 by one FFMA whose
// rounding lands the bucket index in the low mantissa bits, the bucket holds at
// most one decision midpoint, and one compare finishes the search.  The fp32
// rotation differs from the exact value by at most ~7.5e-6 (seven rounded
// additions of terms whose magnitudes sum to <= sqrt(128), plus the scaling), so
// every element that lands within 1e-5 of a midpoint is re-decided exactly: the
// warp recomputes that one rotated value in fp64 from the original weights
// (32 lanes x 4 terms, shuffle reduction) and compares it with the fp64
// midpoints.  The norm is treated the same way: the fp32 sum of squares is
// accurate to ~1e-6, and a block whose norm lies that close to a binary16
// rounding midpoint gets its norm recomputed in fp64 by the warp.  The result is
// the exact nearest-centroid encoding of the exactly rotated block.
//
// Dequantizer ("Qwopus3.6-27B-v2 . HLWQ Q5", Pipeline: dequantize per-Linear):
// the inverse is the same rotation (H symmetric, H H = 128 I): one thread per
// block looks up the 128 centroids, runs the in-register butterflies and scales
// by n16 / 128.

#include "hlwq_common.cuh"

namespace hlwq {

namespace {

constexpr int kBuckets = 2048;
constexpr float kGuard = 1e-5f;
// 1.5 * 2^23 + 768: fmaf(y, 64, kMagic) leaves round(64 y + 768) in the low
// mantissa bits for |64 y + 768| < 2^22.
constexpr float kMagic = 12583680.0f;
constexpr int kQuantThreads = 128;

struct QuantSmem {
  float2 bucket[kBuckets];  // {threshold (shifted domain), base code as int bits}
  double mid[kLevels - 1];  // exact decision midpoints (fp64)
  float sigma;              // grid shift, see build_quant_tables
};

// All-15 code pattern (code of y = 0 under ties-to-lower): 128 fields of 0b01111.
__host__ __device__ constexpr uint32_t code15_word(int w) {
  uint32_t r = 0;
  for (int bit = 0; bit < 32; ++bit) {
    const int gbit = w * 32 + bit;
    if ((gbit % 5) < 4) r |= 1u << bit;
  }
  return r;
}

// Builds the shifted bucket table.  A shift sigma (a multiple of 1/1024) is
// chosen so that no midpoint lies within 4e-5 of a bucket edge; then a value
// and its exact counterpart, which differ by < 1e-5, always fall in buckets
// that give the same code unless the bucket's own midpoint is within the guard
// band (checked per element).  If no shift works (not the case for a Lloyd-Max
// codebook), buckets near an edge get a NaN threshold, which sends every
// element landing there to the exact path.
__device__ void build_quant_tables(QuantSmem& s, const float* __restrict__ codebook) {
  const int tid = threadIdx.x;
  if (tid < kLevels - 1) {
    const float a = __ldg(codebook + tid), b = __ldg(codebook + tid + 1);
    s.mid[tid] = 0.5 * (static_cast<double>(a) + static_cast<double>(b));
    if (!(a < b) || !isfinite(a) || !isfinite(b)) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
  __syncthreads();
  if (tid < 32) {
    const double sig = tid < 16 ? tid * (1.0 / 1024.0) : 0.0;
    bool ok = tid < 16;
    for (int k = 0; k < kLevels - 1 && ok; ++k) {
      const double p = 64.0 * (s.mid[k] + sig) + 768.0;
      const double frac = p - floor(p);
      if (fabs(frac - 0.5) < 64.0 * 4e-5) ok = false;
    }
    const unsigned good = __ballot_sync(0xffffffffu, ok);
    if (tid == 0) s.sigma = good ? static_cast<float>((__ffs(good) - 1) * (1.0 / 1024.0)) : -1.0f;
  }
  __syncthreads();
  const bool shifted = s.sigma >= 0.0f;
  const double sig = shifted ? static_cast<double>(s.sigma) : 0.0;
  for (int i = tid; i < kBuckets; i += blockDim.x) {
    const double lo = (i - 768.5) / 64.0, hi = (i - 767.5) / 64.0;
    int below = 0, inside = 0, inside_k = -1;
    bool risky = false;
    for (int k = 0; k < kLevels - 1; ++k) {
      const double m = s.mid[k] + sig;
      if (m < lo) ++below;
      else if (m <= hi) { ++inside; inside_k = k; }
      if (!shifted && (fabs(m - lo) < 4e-5 || fabs(m - hi) < 4e-5)) risky = true;
    }
    float thr;
    if (inside >= 2 || risky) thr = __int_as_float(0x7fc00000);  // NaN -> always exact path
    else if (inside == 1) thr = static_cast<float>(s.mid[inside_k] + sig);
    else thr = 3.0e38f;
    s.bucket[i] = make_float2(thr, __int_as_float(below));
  }
  if (tid == 0 && !shifted) s.sigma = 0.0f;
  __syncthreads();
}

template <int H>
__device__ __forceinline__ void butterfly_stage(float (&v)[kBlock]) {
#pragma unroll
  for (int i = 0; i < kBlock; ++i) {
    if ((i & H) == 0) {
      const float a = v[i], b = v[i + H];
      v[i] = a + b;
      v[i + H] = a - b;
    }
  }
}

// In-place unnormalised Walsh-Hadamard transform in natural (Sylvester) order:
// v <- v @ H with H[i][j] = (-1)^popcount(i & j).
__device__ __forceinline__ void fwht128(float (&v)[kBlock]) {
  butterfly_stage<1>(v);
  butterfly_stage<2>(v);
  butterfly_stage<4>(v);
  butterfly_stage<8>(v);
  butterfly_stage<16>(v);
  butterfly_stage<32>(v);
  butterfly_stage<64>(v);
}

// Loads one (possibly partial) block into registers, zero-padded.
template <bool kBf16, bool kVec>
__device__ __forceinline__ void load_block(const void* __restrict__ base, int len, float (&v)[kBlock]) {
  if constexpr (kVec && kBf16) {
    const uint4* p = static_cast<const uint4*>(base);
#pragma unroll
    for (int q = 0; q < 16; ++q) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (8 * q < len) u = ldg_stream(p + q);
      v[8 * q + 0] = bf16x2_lo(u.x); v[8 * q + 1] = bf16x2_hi(u.x);
      v[8 * q + 2] = bf16x2_lo(u.y); v[8 * q + 3] = bf16x2_hi(u.y);
      v[8 * q + 4] = bf16x2_lo(u.z); v[8 * q + 5] = bf16x2_hi(u.z);
      v[8 * q + 6] = bf16x2_lo(u.w); v[8 * q + 7] = bf16x2_hi(u.w);
    }
  } else if constexpr (kVec && !kBf16) {
    const uint4* p = static_cast<const uint4*>(base);
#pragma unroll
    for (int q = 0; q < 32; ++q) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (4 * q < len) u = ldg_stream(p + q);
      v[4 * q + 0] = __uint_as_float(u.x); v[4 * q + 1] = __uint_as_float(u.y);
      v[4 * q + 2] = __uint_as_float(u.z); v[4 * q + 3] = __uint_as_float(u.w);
    }
  } else {
#pragma unroll
    for (int j = 0; j < kBlock; ++j) {
      float f = 0.0f;
      if (j < len) {
        if constexpr (kBf16) f = bf16_bits_to_float(__ldg(static_cast<const uint16_t*>(base) + j));
        else f = __ldg(static_cast<const float*>(base) + j);
      }
      v[j] = f;
    }
  }
}

// Element i of a block in fp64 (original input, for the exact path).
template <bool kBf16>
__device__ __forceinline__ double load_elem64(const void* base, int i, int len) {
  if (i >= len) return 0.0;
  if constexpr (kBf16) return static_cast<double>(bf16_bits_to_float(static_cast<const uint16_t*>(base)[i]));
  else return static_cast<double>(static_cast<const float*>(base)[i]);
}

__device__ __forceinline__ double warp_sum64(double x) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) x += __shfl_xor_sync(0xffffffffu, x, off);
  return x;
}

// Replaces the 5-bit field of code j in the 640-bit block held in p[20].
__device__ __forceinline__ void patch_code(uint32_t (&p)[20], int j, uint32_t code) {
  const int bit = 5 * j, w = bit >> 5, sh = bit & 31;
#pragma unroll
  for (int q = 0; q < 20; ++q) {
    if (q == w) p[q] = (p[q] & ~(31u << sh)) | (code << sh);
    if (q == w + 1 && sh > 27) {
      const int hb = sh - 27;  // bits that spill into the next word
      p[q] = (p[q] & ~((1u << hb) - 1u)) | (code >> (5 - hb));
    }
  }
}

template <bool kBf16, bool kVec>
__global__ void __launch_bounds__(kQuantThreads, 3)
quantize_kernel(const void* __restrict__ W, int64_t rows, int in, int nb,
                const float* __restrict__ codebook, uint8_t* __restrict__ packed,
                uint16_t* __restrict__ norms) {
  __shared__ QuantSmem s;
  build_quant_tables(s, codebook);
  const float sigma = s.sigma;
  constexpr int kEsz = kBf16 ? 2 : 4;

  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kQuantThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kQuantThreads / 32);
  const int64_t nblocks = rows * nb;

  for (int64_t first = warp * 32; first < nblocks; first += nwarps * 32) {
    const int64_t F = first + lane;
    const bool active = F < nblocks;
    int64_t o = 0;
    int b = 0, len = 0;
    const char* wblk = static_cast<const char*>(W);
    if (active) {
      o = F / nb;
      b = static_cast<int>(F - o * nb);
      len = min(kBlock, in - kBlock * b);
      wblk += (o * static_cast<int64_t>(in) + static_cast<int64_t>(kBlock) * b) * kEsz;
    }

    float v[kBlock];
    load_block<kBf16, kVec>(wblk, active ? len : 0, v);

    float acc[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
#pragma unroll
    for (int j = 0; j < kBlock; ++j) acc[j & 7] = fmaf(v[j], v[j], acc[j & 7]);
    float ssum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));

    bool zero_block = false, norm_exact = false;
    if (!(ssum >= 0x1p-100f && ssum <= 0x1p100f)) {
      // Zero, tiny, huge or non-finite block: rescale by a power of two (codes
      // are scale-invariant) and take the norm on the exact path.
      float mx = 0.0f;
#pragma unroll
      for (int j = 0; j < kBlock; ++j) mx = fmaxf(mx, fabsf(v[j]));
      if (mx == 0.0f) {
        zero_block = true;
      } else if (isfinite(mx)) {
        int e;
        frexpf(mx, &e);
        const float sc = ldexpf(1.0f, -e);
#pragma unroll
        for (int j = 0; j < kBlock; ++j) v[j] *= sc;
#pragma unroll
        for (int k = 0; k < 8; ++k) acc[k] = 0.0f;
#pragma unroll
        for (int j = 0; j < kBlock; ++j) acc[j & 7] = fmaf(v[j], v[j], acc[j & 7]);
        ssum = ((acc[0] + acc[1]) + (acc[2] + acc[3])) + ((acc[4] + acc[5]) + (acc[6] + acc[7]));
      }
      norm_exact = active && !zero_block;
    }
    const float n32 = sqrtf(ssum);
    uint16_t h16 = zero_block ? 0 : __half_as_ushort(__float2half_rn(n32));
    if (!norm_exact && active && !zero_block) {
      // Norm within ~2e-6 relative of a binary16 rounding midpoint -> exact path.
      const uint16_t lo16 = __half_as_ushort(__float2half_rn(n32 * (1.0f - 2e-6f)));
      const uint16_t hi16 = __half_as_ushort(__float2half_rn(n32 * (1.0f + 2e-6f)));
      norm_exact = lo16 != hi16;
    }
    const float inv = zero_block ? 0.0f : 1.0f / n32;

    uint32_t p[20];
    uint32_t fm[4] = {0u, 0u, 0u, 0u};
    if (zero_block || !active) {
#pragma unroll
      for (int w = 0; w < 20; ++w) p[w] = code15_word(w);
    } else {
      fwht128(v);
#pragma unroll
      for (int w = 0; w < 20; ++w) p[w] = 0u;
#pragma unroll
      for (int j = 0; j < kBlock; ++j) {
        const float ys = fmaf(v[j], inv, sigma);
        const float tf = fmaf(ys, 64.0f, kMagic);
        const float2 e = s.bucket[__float_as_uint(tf) & (kBuckets - 1)];
        const uint32_t code = static_cast<uint32_t>(__float_as_int(e.y)) + (ys > e.x ? 1u : 0u);
        if (!(fabsf(ys - e.x) >= kGuard)) fm[j >> 5] |= 1u << (j & 31);
        const int bit = 5 * j, w = bit >> 5, sh = bit & 31;
        p[w] |= code << sh;
        if (sh > 27) p[w + 1] |= code >> (32 - sh);
      }
    }

    // Exact path for norms near a binary16 rounding midpoint.
    for (unsigned bal = __ballot_sync(0xffffffffu, norm_exact); bal; bal &= bal - 1) {
      const int src = __ffs(bal) - 1;
      const char* base = reinterpret_cast<const char*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(wblk), src));
      const int slen = __shfl_sync(0xffffffffu, len, src);
      double q = 0.0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const double w = load_elem64<kBf16>(base, lane + 32 * t, slen);
        q = fma(w, w, q);
      }
      q = warp_sum64(q);
      if (lane == src) h16 = __half_as_ushort(__double2half(sqrt(q)));
    }

    // Exact path for codes within the guard band of a midpoint.
    for (;;) {
      const unsigned bal = __ballot_sync(0xffffffffu, (fm[0] | fm[1] | fm[2] | fm[3]) != 0u);
      if (!bal) break;
      const int src = __ffs(bal) - 1;
      int jl = 0;
      if (lane == src) {
        if (fm[0]) jl = __ffs(fm[0]) - 1;
        else if (fm[1]) jl = 32 + __ffs(fm[1]) - 1;
        else if (fm[2]) jl = 64 + __ffs(fm[2]) - 1;
        else jl = 96 + __ffs(fm[3]) - 1;
      }
      const int j = __shfl_sync(0xffffffffu, jl, src);
      const char* base = reinterpret_cast<const char*>(
          __shfl_sync(0xffffffffu, reinterpret_cast<unsigned long long>(wblk), src));
      const int slen = __shfl_sync(0xffffffffu, len, src);
      double sy = 0.0, q = 0.0;
#pragma unroll
      for (int t = 0; t < 4; ++t) {
        const int i = lane + 32 * t;
        const double w = load_elem64<kBf16>(base, i, slen);
        q = fma(w, w, q);
        sy += (__popc(i & j) & 1) ? -w : w;
      }
      sy = warp_sum64(sy);
      q = warp_sum64(q);
      const double y = q > 0.0 ? sy / sqrt(q) : 0.0;
      uint32_t code = 0;
#pragma unroll
      for (int k = 0; k < kLevels - 1; ++k) code += (y > s.mid[k]) ? 1u : 0u;
      if (lane == src) {
        patch_code(p, j, code);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q == (j >> 5)) fm[q] &= ~(1u << (j & 31));
      }
    }

    if (active) {
      uint4* dst = reinterpret_cast<uint4*>(packed + F * kBlockBytes);
#pragma unroll
      for (int q = 0; q < 5; ++q) dst[q] = make_uint4(p[4 * q], p[4 * q + 1], p[4 * q + 2], p[4 * q + 3]);
      norms[F] = h16;
    }
  }
}

// ---------------------------------------------------------------- dequantize
constexpr int kDequantThreads = 128;

template <bool kOutBf16, bool kVec>
__global__ void __launch_bounds__(kDequantThreads, 3)
dequantize_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                  const float* __restrict__ codebook, int64_t rows, int in, int nb,
                  void* __restrict__ out) {
  __shared__ float cb[kLevels];
  if (threadIdx.x < kLevels) cb[threadIdx.x] = __ldg(codebook + threadIdx.x);
  __syncthreads();
  const int64_t nblocks = rows * nb;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * kDequantThreads;
  for (int64_t F = static_cast<int64_t>(blockIdx.x) * kDequantThreads + threadIdx.x; F < nblocks; F += stride) {
    const int64_t o = F / nb;
    const int b = static_cast<int>(F - o * nb);
    const int len = min(kBlock, in - kBlock * b);
    uint32_t w[20];
    const uint4* src = reinterpret_cast<const uint4*>(packed + F * kBlockBytes);
#pragma unroll
    for (int q = 0; q < 5; ++q) {
      const uint4 u = ldg_stream(src + q);
      w[4 * q] = u.x; w[4 * q + 1] = u.y; w[4 * q + 2] = u.z; w[4 * q + 3] = u.w;
    }
    float v[kBlock];
#pragma unroll
    for (int j = 0; j < kBlock; ++j) {
      const int bit = 5 * j, q = bit >> 5, sh = bit & 31;
      uint32_t code;
      if (sh <= 27) code = (w[q] >> sh) & 31u;
      else code = __funnelshift_r(w[q], w[q + 1], sh) & 31u;
      v[j] = cb[code];
    }
    fwht128(v);
    const float scale = half_bits_to_float(__ldg(norms + F)) * (1.0f / 128.0f);
    const int64_t off = o * static_cast<int64_t>(in) + static_cast<int64_t>(kBlock) * b;
    if constexpr (!kOutBf16) {
      float* dst = static_cast<float*>(out) + off;
      if constexpr (kVec) {
#pragma unroll
        for (int q = 0; q < 32; ++q)
          if (4 * q < len)
            reinterpret_cast<float4*>(dst)[q] =
                make_float4(v[4 * q] * scale, v[4 * q + 1] * scale, v[4 * q + 2] * scale, v[4 * q + 3] * scale);
      } else {
#pragma unroll
        for (int j = 0; j < kBlock; ++j)
          if (j < len) dst[j] = v[j] * scale;
      }
    } else {
      uint16_t* dst = static_cast<uint16_t*>(out) + off;
      if constexpr (kVec) {
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          if (8 * q < len) {
            uint4 u;
            u.x = float_to_bf16_bits(v[8 * q] * scale) | (float_to_bf16_bits(v[8 * q + 1] * scale) << 16);
            u.y = float_to_bf16_bits(v[8 * q + 2] * scale) | (float_to_bf16_bits(v[8 * q + 3] * scale) << 16);
            u.z = float_to_bf16_bits(v[8 * q + 4] * scale) | (float_to_bf16_bits(v[8 * q + 5] * scale) << 16);
            u.w = float_to_bf16_bits(v[8 * q + 6] * scale) | (float_to_bf16_bits(v[8 * q + 7] * scale) << 16);
            reinterpret_cast<uint4*>(dst)[q] = u;
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < kBlock; ++j)
          if (j < len) dst[j] = static_cast<uint16_t>(float_to_bf16_bits(v[j] * scale));
      }
    }
  }
}

}  // namespace

int launch_quantize(const void* W, bool bf16, int64_t rows, int in, const float* codebook,
                    uint8_t* packed, uint16_t* norms, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int64_t nblocks = rows * nb;
  const int64_t warps_needed = ceil_div(nblocks, 32);
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 3;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(warps_needed, kQuantThreads / 32)));
  const bool vec = (reinterpret_cast<uintptr_t>(W) % 16 == 0) &&
                   ((static_cast<int64_t>(in) * (bf16 ? 2 : 4)) % 16 == 0);
  if (bf16) {
    if (vec) quantize_kernel<true, true><<<grid, kQuantThreads, 0, stream>>>(W, rows, in, nb, codebook, packed, norms);
    else quantize_kernel<true, false><<<grid, kQuantThreads, 0, stream>>>(W, rows, in, nb, codebook, packed, norms);
  } else {
    if (vec) quantize_kernel<false, true><<<grid, kQuantThreads, 0, stream>>>(W, rows, in, nb, codebook, packed, norms);
    else quantize_kernel<false, false><<<grid, kQuantThreads, 0, stream>>>(W, rows, in, nb, codebook, packed, norms);
  }
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t rows,
                      int in, void* out, bool bf16, cudaStream_t stream) {
  const int nb = static_cast<int>(ceil_div(in, kBlock));
  const int64_t nblocks = rows * nb;
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 3;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(nblocks, kDequantThreads)));
  const bool vec = (reinterpret_cast<uintptr_t>(out) % 16 == 0) &&
                   ((static_cast<int64_t>(in) * (bf16 ? 2 : 4)) % 16 == 0);
  if (bf16) {
    if (vec) dequantize_kernel<true, true><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
    else dequantize_kernel<true, false><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
  } else {
    if (vec) dequantize_kernel<false, true><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
    else dequantize_kernel<false, false><<<grid, kDequantThreads, 0, stream>>>(packed, norms, codebook, rows, in, nb, out);
  }
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace hlwq
