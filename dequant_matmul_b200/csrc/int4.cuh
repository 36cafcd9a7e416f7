#pragma once
// HLWQ Q5 -> INT4 re-encoder (sm_100a).
//
// "Qwopus3.6-27B-v2 . HLWQ Q5", Pipeline: the Q5 weights are dequantized per
// Linear and re-encoded as INT4 weight-only with groups of 128 on the
// 128-aligned Linears.  Per row and group (= Q5 block) b:
//   w     = n16 / 128 * sum_j c[k_j] H[j][i]           (the Q5 dequantization)
//   s     = bf16((max w - min w) / 15),  z = bf16(min w + 0)  (a zero minimum -> +0)
//   q_i   = clamp(rint((w_i - z) / s), 0, 15)          (0 when s = 0)
// stored two codes per byte (element 2k in the low nibble of byte k), 64 bytes
// per group, s and z as bfloat16 bit patterns.
//
// Exactness.  w is exact in fp64: 128 fp32 centroids summed with signs (at
// most ~37 significant bits), times the fp16 norm over 128.  The kernel
// evaluates every step in fp64, so min, max, s, z and the rounded quotients
// are those of any fp64 evaluation of the same formulas.  The quotient is
// formed as (w - z) * (1 / s); where that product lies within 8 ulps of a
// half-way point the exact fp64 division decides, so every code equals
// rint(fl((w - z) / s)).  bf16 values are rounded to nearest even directly
// from the fp64 bit pattern (no intermediate fp32); magnitudes below 2^-126
// give a signed zero.
//
// Fast path and exact path.  The block is first rotated and encoded in fp32.
// The fp32 rotation is within E = 10 * 2^-24 * sum_j |c[k_j]| * n16 / 128 of
// the exact weights (7 rounded butterfly stages whose partial sums are bounded
// by sum |c|, plus the scaling), so the fp32 results are certain when s and z
// round to the same bfloat16 for every value within that bound, and every
// quotient lies farther than E / s + 4e-6 from a half-way point.  A block
// that fails these checks is marked (its scale set to 0xffff, a bfloat16 NaN
// that no block's scale can be) and left to a second kernel, which gathers the
// marked blocks eight per warp and takes the exact path for each (every step
// in fp64, the quotient as (w - z) * (1 / s) with the division where that
// product lies within 8 ulps of a half-way point).  About 0.2 % of the blocks
// of a layer are marked, so the fp64 work is that small share.
//
// Layout as the dequantizer: four lanes per 128-block, 32 values each; the
// inverse rotation is 5 register butterfly stages and 2 shuffle stages.

#include "hlwq_common.cuh"
#include "quantize.cuh"

namespace hlwq {

namespace {

constexpr int kI4Threads = 256;
constexpr int kI4GroupBytes = kBlock / 2;  // 64
constexpr uint16_t kI4Unsure = 0xffffu;      // scale mark of a block left to the exact path

// bfloat16 bits of a finite fp64 value, round to nearest even.
__device__ __forceinline__ uint32_t bf16_rne_from_f64(double x) {
  const uint64_t bits = static_cast<uint64_t>(__double_as_longlong(x));
  const uint32_t sign = static_cast<uint32_t>(bits >> 48) & 0x8000u;
  const uint64_t a = bits & 0x7fffffffffffffffull;
  if (a < 0x3810000000000000ull) return sign;  // |x| < 2^-126
  const uint64_t r = a + 0x00000fffffffffffull + ((a >> 45) & 1ull);  // round the 52-bit mantissa to 7 bits
  const int e8 = static_cast<int>(r >> 52) - 1023 + 127;
  return sign | (static_cast<uint32_t>(e8) << 7) | (static_cast<uint32_t>(r >> 45) & 0x7fu);
}

__device__ __forceinline__ double bf16_bits_to_f64(uint32_t b) {
  return static_cast<double>(__uint_as_float(b << 16));
}

template <int H>
__device__ __forceinline__ void stage32_f64(double (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if ((i & H) == 0) {
      const double a = v[i], c = v[i + H];
      v[i] = a + c;
      v[i + H] = a - c;
    }
}

// values 32 * LM apart live in lanes LM apart: the lower lane keeps a + b,
// the upper one b - a
template <int LM>
__device__ __forceinline__ void stage_x_f64(double (&v)[32], int lane) {
  const bool upper = (lane & LM) != 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const double p = __shfl_xor_sync(0xffffffffu, v[i], LM);
    v[i] = upper ? p - v[i] : v[i] + p;
  }
}

__device__ __forceinline__ float quad_min_f32(float x) {
  x = fminf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fminf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ float quad_max_f32(float x) {
  x = fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmaxf(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ double quad_min_f64(double x) {
  x = fmin(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmin(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__device__ __forceinline__ double quad_max_f64(double x) {
  x = fmax(x, __shfl_xor_sync(0xffffffffu, x, 1));
  return fmax(x, __shfl_xor_sync(0xffffffffu, x, 2));
}

__global__ void __launch_bounds__(kI4Threads)
requantize_int4_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                       const float* __restrict__ codebook, int64_t nblocks, uint8_t* __restrict__ q4,
                       uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  __shared__ float cb32[kLevels];
  if (threadIdx.x < kLevels) cb32[threadIdx.x] = __ldg(codebook + threadIdx.x);
  __syncthreads();
  const int lane = threadIdx.x & 31, q = lane & 3;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kI4Threads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kI4Threads / 32);
  for (int64_t first = warp * 8; first < nblocks; first += nwarps * 8) {
    const int64_t F = first + (lane >> 2);
    const bool active = F < nblocks;
    uint32_t w[5] = {0u, 0u, 0u, 0u, 0u};
    double nsc = 0.0;
    if (active) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + F * kBlockBytes + 20 * q);
#pragma unroll
      for (int k = 0; k < 5; ++k) w[k] = __ldg(src + k);
      nsc = static_cast<double>(half_bits_to_float(__ldg(norms + F))) * (1.0 / 128.0);
    }
    uint32_t code5[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const int bit = 5 * e, k = bit >> 5, sh = bit & 31;
      code5[e] = (sh <= 27) ? ((w[k] >> sh) & 31u) : (__funnelshift_r(w[k], w[k + 1], sh) & 31u);
    }
    uint32_t s16, z16, out[4] = {0u, 0u, 0u, 0u};
    // ---- fast path (fp32) with the checks that make its results exact
    bool sure = true;
    {
      float v[32];
      float asum = 0.0f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        v[e] = cb32[code5[e]];
        asum += fabsf(v[e]);
      }
      asum = quad_sum(asum);
      fwht_4lanes(v, lane);
      const float nscf = static_cast<float>(nsc);  // n16 / 128: exact in fp32
      float lo = 3.0e38f, hi = -3.0e38f;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        v[e] *= nscf;
        lo = fminf(lo, v[e]);
        hi = fmaxf(hi, v[e]);
      }
      lo = quad_min_f32(lo);
      hi = quad_max_f32(hi);
      const double err = 10.0 * 5.9604644775390625e-8 * static_cast<double>(asum) * nsc;
      const double S = (static_cast<double>(hi) - static_cast<double>(lo)) / 15.0;
      const double dS = 2.0 * err / 15.0 * 1.01 + 1e-15 * fabs(S);
      const double L = static_cast<double>(lo);
      s16 = bf16_rne_from_f64(S);
      z16 = bf16_rne_from_f64(__dadd_rn(L, 0.0));
      sure = bf16_rne_from_f64(S - dS) == s16 && bf16_rne_from_f64(S + dS) == s16 &&
             bf16_rne_from_f64(__dadd_rn(L - err, 0.0)) == z16 && bf16_rne_from_f64(__dadd_rn(L + err, 0.0)) == z16;
      const float sf = __uint_as_float(s16 << 16), zf = __uint_as_float(z16 << 16);
      if (sf > 0.0f) {
        const float rsf = 1.0f / sf;
        const float band = static_cast<float>(err / static_cast<double>(sf)) + 4e-6f;
#pragma unroll
        for (int e = 0; e < 32; ++e) {
          const float t = (v[e] - zf) * rsf;
          if (fabsf(t - floorf(t) - 0.5f) <= band) sure = false;
          const uint32_t code = static_cast<uint32_t>(fminf(fmaxf(rintf(t), 0.0f), 15.0f));
          out[e >> 3] |= code << (4 * (e & 7));
        }
      }
    }
    // the quad's verdict: every lane of the block must be sure
    sure = __shfl_xor_sync(0xffffffffu, sure, 1) && sure;
    sure = __shfl_xor_sync(0xffffffffu, sure, 2) && sure;
    if (active && sure) {
      *reinterpret_cast<uint4*>(q4 + F * kI4GroupBytes + 16 * q) = make_uint4(out[0], out[1], out[2], out[3]);
      if (q == 0) {
        scale[F] = static_cast<uint16_t>(s16);
        zero[F] = static_cast<uint16_t>(z16);
      }
    } else if (active && q == 0) {
      scale[F] = kI4Unsure;  // the exact kernel takes this block
    }
  }
}

// The exact path for the blocks the fast kernel marked: a warp looks at 32
// consecutive blocks, gathers the marked ones and encodes them eight at a
// time (one block per quad of lanes), every step in fp64.
__global__ void __launch_bounds__(kI4Threads)
requantize_int4_exact_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                             const float* __restrict__ codebook, int64_t nblocks, uint8_t* __restrict__ q4,
                             uint16_t* __restrict__ scale, uint16_t* __restrict__ zero) {
  __shared__ float cb32[kLevels];
  if (threadIdx.x < kLevels) cb32[threadIdx.x] = __ldg(codebook + threadIdx.x);
  __syncthreads();
  const int lane = threadIdx.x & 31, q = lane & 3, quad = lane >> 2;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kI4Threads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kI4Threads / 32);
  for (int64_t first = warp * 32; first < nblocks; first += nwarps * 32) {
    const int64_t mine = first + lane;
    uint32_t marked = __ballot_sync(0xffffffffu, mine < nblocks && scale[mine] == kI4Unsure);
    while (marked) {
      // the quad takes the quad-th marked block of this round (if any)
      uint32_t m = marked;
      for (int k = 0; k < quad && m; ++k) m &= m - 1;
      const bool active = m != 0u;
      const int64_t F = active ? first + (__ffs(m) - 1) : first;
      for (int k = 0; k < 8 && marked; ++k) marked &= marked - 1;  // eight blocks per round
      uint32_t w[5] = {0u, 0u, 0u, 0u, 0u};
      double nsc = 0.0;
      if (active) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + F * kBlockBytes + 20 * q);
#pragma unroll
        for (int k = 0; k < 5; ++k) w[k] = __ldg(src + k);
        nsc = static_cast<double>(half_bits_to_float(__ldg(norms + F))) * (1.0 / 128.0);
      }
      double v[32];
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        const int bit = 5 * e, k = bit >> 5, sh = bit & 31;
        const uint32_t c = (sh <= 27) ? ((w[k] >> sh) & 31u) : (__funnelshift_r(w[k], w[k + 1], sh) & 31u);
        v[e] = static_cast<double>(cb32[c]);
      }
      stage32_f64<1>(v);
      stage32_f64<2>(v);
      stage32_f64<4>(v);
      stage32_f64<8>(v);
      stage32_f64<16>(v);
      stage_x_f64<1>(v, lane);
      stage_x_f64<2>(v, lane);
      double lo = 1.0e300, hi = -1.0e300;
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        v[e] *= nsc;  // exact: the Q5 dequantized weight
        lo = fmin(lo, v[e]);
        hi = fmax(hi, v[e]);
      }
      lo = quad_min_f64(lo);
      hi = quad_max_f64(hi);
      const uint32_t s16 = bf16_rne_from_f64((hi - lo) / 15.0);
      const uint32_t z16 = bf16_rne_from_f64(__dadd_rn(lo, 0.0));  // a zero minimum is stored as +0
      const double sv = bf16_bits_to_f64(s16), z = bf16_bits_to_f64(z16);
      const double rs = sv > 0.0 ? 1.0 / sv : 0.0;
      uint32_t out[4] = {0u, 0u, 0u, 0u};
#pragma unroll
      for (int e = 0; e < 32; ++e) {
        uint32_t code = 0u;
        if (sv > 0.0) {
          const double d = v[e] - z;
          double t = d * rs;
          // within 8 ulps of a half-way point: the division decides
          const double f = t - floor(t);
          if (fabs(f - 0.5) <= 8.0 * 2.220446049250313e-16 * fmax(fabs(t), 1.0)) t = d / sv;
          code = static_cast<uint32_t>(fmin(fmax(rint(t), 0.0), 15.0));
        }
        out[e >> 3] |= code << (4 * (e & 7));
      }
      if (active) {
        *reinterpret_cast<uint4*>(q4 + F * kI4GroupBytes + 16 * q) = make_uint4(out[0], out[1], out[2], out[3]);
        if (q == 0) {
          zero[F] = static_cast<uint16_t>(z16);
          scale[F] = static_cast<uint16_t>(s16);
        }
      }
    }
  }
}

}  // namespace

int launch_requantize_int4(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t rows,
                           int in, uint8_t* q4, uint16_t* scale, uint16_t* zero, cudaStream_t stream) {
  const int64_t nblocks = rows * (in / kBlock);
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(nblocks, kI4Threads / 4)));
  requantize_int4_kernel<<<grid, kI4Threads, 0, stream>>>(packed, norms, codebook, nblocks, q4, scale, zero);
  if (cudaGetLastError() != cudaSuccess) return HLWQ_ECUDA;
  const int grid2 = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(nblocks, kI4Threads)));
  requantize_int4_exact_kernel<<<grid2, kI4Threads, 0, stream>>>(packed, norms, codebook, nblocks, q4, scale, zero);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

}  // namespace hlwq
