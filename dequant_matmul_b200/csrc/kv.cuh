#pragma once
// HLWQ Q3 KV-cache encoding (sm_100a): per-head 256-value vectors, 8-level
// Lloyd-Max codes, 3 bits per value ("Qwopus3.6-27B-v2 . HLWQ Q5",
// "Methodology notes", KV-cache bullet; head_dim = 256).
//
//   quantize    n = ||x||_2 -> fp16; y = (x @ H256) / n; code_j = number of
//               decision midpoints below y_j (nearest centroid, ties low);
//               code j at bits [3j, 3j + 3) of the vector's 96 bytes.
//   dequantize  x_hat = n16 * (c[code] @ H256) / 256.
//   scores      s[m][i] = q_m . x_hat_i = (n16_i / 256) sum_j c[k_ij] (q_m @ H256)_j,
//               evaluated in the rotated domain: each query is rotated once.
//
// Layout: eight lanes per vector, 32 consecutive values each, four vectors per
// warp; the rotation is 5 butterfly stages in registers and 3 shuffle stages
// (lane xor 1, 2, 4).  The quantizer works in fp64: the +-1 sums of bf16
// values are exact there, and the norm, the division by it and the midpoint
// comparisons are the correctly rounded fp64 operations of the definition, so
// the codes and norms are those of an fp64 evaluation.  The fp16 norm is
// rounded to nearest even directly from fp64.  Dequantizer and scores work in
// fp32.

#include "hlwq_common.cuh"

namespace hlwq {

namespace {

constexpr int kKvDim = 256;
constexpr int kKvBytes = 96;
constexpr int kKvLevels = 8;
constexpr int kKvThreads = 256;
constexpr int kKvMaxQueries = 64;  // queries per scores launch (rotated copies in shared memory)

// binary16 bits of a finite, non-negative fp64 value, round to nearest even.
__device__ __forceinline__ uint32_t f16_rne_from_f64(double v) {
  if (!(v > 0.0)) return 0u;
  if (v >= 65520.0) return 0x7c00u;                        // rounds to infinity
  if (v < 6.103515625e-05) return static_cast<uint32_t>(rint(v * 16777216.0));  // subnormal: units of 2^-24
  int e;
  const double m = frexp(v, &e);                           // v = m 2^e, m in [0.5, 1)
  double sig = rint(m * 2048.0);                           // 11 significant bits
  if (sig == 2048.0) {
    sig = 1024.0;
    ++e;
  }
  const int e5 = e - 1 + 15;
  if (e5 >= 31) return 0x7c00u;
  return (static_cast<uint32_t>(e5) << 10) | (static_cast<uint32_t>(sig) - 1024u);
}

template <typename T, int H>
__device__ __forceinline__ void kv_stage(T (&v)[32]) {
#pragma unroll
  for (int i = 0; i < 32; ++i)
    if ((i & H) == 0) {
      const T a = v[i], c = v[i + H];
      v[i] = a + c;
      v[i + H] = a - c;
    }
}

template <typename T, int LM>
__device__ __forceinline__ void kv_stage_x(T (&v)[32], int lane) {
  const bool upper = (lane & LM) != 0;
#pragma unroll
  for (int i = 0; i < 32; ++i) {
    const T p = __shfl_xor_sync(0xffffffffu, v[i], LM);
    v[i] = upper ? p - v[i] : v[i] + p;
  }
}

// The 256-point transform of the vector held by 8 lanes (32 values each).
template <typename T>
__device__ __forceinline__ void kv_fwht(T (&v)[32], int lane) {
  kv_stage<T, 1>(v);
  kv_stage<T, 2>(v);
  kv_stage<T, 4>(v);
  kv_stage<T, 8>(v);
  kv_stage<T, 16>(v);
  kv_stage_x<T, 1>(v, lane);
  kv_stage_x<T, 2>(v, lane);
  kv_stage_x<T, 4>(v, lane);
}

template <typename T>
__device__ __forceinline__ T oct_sum(T x) {
  x += __shfl_xor_sync(0xffffffffu, x, 1);
  x += __shfl_xor_sync(0xffffffffu, x, 2);
  return x + __shfl_xor_sync(0xffffffffu, x, 4);
}

// 3-bit field of code e (0..31) in a lane's 96-bit group w[3].
__device__ __forceinline__ uint32_t kv_code(const uint32_t (&w)[3], int e) {
  const int bit = 3 * e, k = bit >> 5, sh = bit & 31;
  return (sh <= 29) ? ((w[k] >> sh) & 7u) : (__funnelshift_r(w[k], w[k + 1], sh) & 7u);
}

__device__ __forceinline__ void kv_check_codebook(const float* cb) {
  if (threadIdx.x + 1 < kKvLevels) {
    const float a = __ldg(cb + threadIdx.x), b = __ldg(cb + threadIdx.x + 1);
    if (!(a < b) || !isfinite(a) || !isfinite(b)) raise_device_error(HLWQ_DEVERR_CODEBOOK);
  }
}

__global__ void __launch_bounds__(kKvThreads)
kv_quantize_kernel(const uint16_t* __restrict__ X, int64_t n, int64_t ldx, const float* __restrict__ codebook,
                   uint8_t* __restrict__ packed, uint16_t* __restrict__ norms, int xvec) {
  __shared__ double mid[kKvLevels - 1];
  kv_check_codebook(codebook);
  if (threadIdx.x < kKvLevels - 1)
    mid[threadIdx.x] = 0.5 * (static_cast<double>(__ldg(codebook + threadIdx.x)) +
                              static_cast<double>(__ldg(codebook + threadIdx.x + 1)));
  __syncthreads();
  const int lane = threadIdx.x & 31, l8 = lane & 7;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kKvThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kKvThreads / 32);
  for (int64_t first = warp * 4; first < n; first += nwarps * 4) {
    const int64_t r = first + (lane >> 3);
    const bool active = r < n;
    double v[32];
    const uint16_t* src = X + (active ? r : 0) * ldx + 32 * l8;
    if (xvec) {
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 u = make_uint4(0u, 0u, 0u, 0u);
        if (active) u = __ldg(reinterpret_cast<const uint4*>(src) + c);
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
        v[e] = active ? static_cast<double>(__uint_as_float(static_cast<uint32_t>(__ldg(src + e)) << 16)) : 0.0;
    }
    double ss = 0.0;
#pragma unroll
    for (int e = 0; e < 32; ++e) ss = fma(v[e], v[e], ss);
    ss = oct_sum(ss);
    const double nrm = sqrt(ss);
    kv_fwht(v, lane);
    uint32_t w[3] = {0u, 0u, 0u};
#pragma unroll
    for (int e = 0; e < 32; ++e) {
      const double y = nrm > 0.0 ? v[e] / nrm : 0.0;
      uint32_t code = 0u;
#pragma unroll
      for (int k = 0; k < kKvLevels - 1; ++k) code += y > mid[k] ? 1u : 0u;
      const int bit = 3 * e, k = bit >> 5, sh = bit & 31;
      w[k] |= code << sh;
      if (sh > 29) w[k + 1] |= code >> (32 - sh);
    }
    if (active) {
      uint32_t* dst = reinterpret_cast<uint32_t*>(packed + r * kKvBytes + 12 * l8);
      dst[0] = w[0];
      dst[1] = w[1];
      dst[2] = w[2];
      if (l8 == 0) norms[r] = static_cast<uint16_t>(f16_rne_from_f64(nrm));
    }
  }
}

template <bool kOutBf16>
__global__ void __launch_bounds__(kKvThreads)
kv_dequantize_kernel(const uint8_t* __restrict__ packed, const uint16_t* __restrict__ norms,
                     const float* __restrict__ codebook, int64_t n, void* __restrict__ out) {
  __shared__ float cb[kKvLevels];
  kv_check_codebook(codebook);
  if (threadIdx.x < kKvLevels) cb[threadIdx.x] = __ldg(codebook + threadIdx.x);
  __syncthreads();
  const int lane = threadIdx.x & 31, l8 = lane & 7;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * kKvThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kKvThreads / 32);
  for (int64_t first = warp * 4; first < n; first += nwarps * 4) {
    const int64_t r = first + (lane >> 3);
    const bool active = r < n;
    uint32_t w[3] = {0u, 0u, 0u};
    float sc = 0.0f;
    if (active) {
      const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + r * kKvBytes + 12 * l8);
      w[0] = __ldg(src);
      w[1] = __ldg(src + 1);
      w[2] = __ldg(src + 2);
      sc = half_bits_to_float(__ldg(norms + r)) * (1.0f / 256.0f);
    }
    float v[32];
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = cb[kv_code(w, e)];
    kv_fwht(v, lane);
    if (!active) continue;
    const int64_t off = r * kKvDim + 32 * l8;
    if constexpr (kOutBf16) {
      uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + off);
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        uint4 u;
        u.x = float_to_bf16_bits(v[8 * c] * sc) | (float_to_bf16_bits(v[8 * c + 1] * sc) << 16);
        u.y = float_to_bf16_bits(v[8 * c + 2] * sc) | (float_to_bf16_bits(v[8 * c + 3] * sc) << 16);
        u.z = float_to_bf16_bits(v[8 * c + 4] * sc) | (float_to_bf16_bits(v[8 * c + 5] * sc) << 16);
        u.w = float_to_bf16_bits(v[8 * c + 6] * sc) | (float_to_bf16_bits(v[8 * c + 7] * sc) << 16);
        dst[c] = u;
      }
    } else {
      float4* dst = reinterpret_cast<float4*>(static_cast<float*>(out) + off);
#pragma unroll
      for (int c = 0; c < 8; ++c)
        dst[c] = make_float4(v[4 * c] * sc, v[4 * c + 1] * sc, v[4 * c + 2] * sc, v[4 * c + 3] * sc);
    }
  }
}

// Rotated queries in shared memory: value p of query m at m * 288 + p + 4 (p / 32),
// so a lane's 32 values are eight aligned 16-byte chunks and the eight lanes of
// a key (positions 32 l8 + j) read disjoint banks with 16-byte loads.
constexpr int kKvQRow = kKvDim + 32;
__host__ __device__ inline int kv_qpos(int m, int p) { return m * kKvQRow + p + 4 * (p >> 5); }

// Scores against the cached keys 0 .. n_total - 1: keys r < n_enc from their
// codes, keys n_enc <= r < n_total exactly from the residual window (bf16 ring
// of R slots, key r in slot r % R), rotated here like the queries, so that
// q . k = (q H) . (k H) / 256 in both cases.
__global__ void __launch_bounds__(kKvThreads)
kv_scores_kernel(const uint16_t* __restrict__ Q, int m_count, int64_t ldq, const uint8_t* __restrict__ packed,
                 const uint16_t* __restrict__ norms, const float* __restrict__ codebook, int64_t n_enc,
                 const uint16_t* __restrict__ window, int64_t R, int64_t n_total, float* __restrict__ S,
                 int64_t lds) {
  extern __shared__ __align__(16) float qs[];  // [m_count][288]
  __shared__ float cb[kKvLevels];
  kv_check_codebook(codebook);
  if (threadIdx.x < kKvLevels) cb[threadIdx.x] = __ldg(codebook + threadIdx.x);
  const int lane = threadIdx.x & 31, l8 = lane & 7, warp = threadIdx.x >> 5;
  // rotate the queries: one 8-lane group per query; the loop is uniform over
  // the warp (the rotation shuffles across all its lanes)
  for (int m0 = warp * 4; m0 < m_count; m0 += (kKvThreads / 32) * 4) {
    const int m = m0 + (lane >> 3);
    const bool mq = m < m_count;
    float v[32];
    const uint16_t* src = Q + static_cast<int64_t>(mq ? m : 0) * ldq + 32 * l8;
#pragma unroll
    for (int e = 0; e < 32; ++e) v[e] = mq ? __uint_as_float(static_cast<uint32_t>(__ldg(src + e)) << 16) : 0.0f;
    kv_fwht(v, lane);
    if (mq) {
#pragma unroll
      for (int e = 0; e < 32; ++e) qs[kv_qpos(m, 32 * l8 + e)] = v[e];
    }
  }
  __syncthreads();
  const int64_t gwarp = (static_cast<int64_t>(blockIdx.x) * kKvThreads + threadIdx.x) >> 5;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kKvThreads / 32);
  for (int64_t first = gwarp * 4; first < n_total; first += nwarps * 4) {
    const int64_t r = first + (lane >> 3);
    const bool active = r < n_total;
    const bool exact = active && r >= n_enc;  // a window key
    float c[32];
    float sc = 0.0f;
    if (__any_sync(0xffffffffu, exact)) {
      // window keys of this warp's four keys (zero for the others), rotated
      // with the queries' butterflies
      float v[32];
      if (exact) {
        const uint4* src = reinterpret_cast<const uint4*>(window + (r % R) * kKvDim + 32 * l8);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          const uint4 u = __ldg(src + k);
          const uint32_t w4[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
          for (int h = 0; h < 4; ++h) {
            v[8 * k + 2 * h] = bf16x2_lo(w4[h]);
            v[8 * k + 2 * h + 1] = bf16x2_hi(w4[h]);
          }
        }
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0.0f;
      }
      kv_fwht(v, lane);
#pragma unroll
      for (int e = 0; e < 32; ++e) c[e] = v[e];
      if (exact) sc = 1.0f / 256.0f;
    }
    if (!exact) {
      uint32_t w[3] = {0u, 0u, 0u};
      if (active) {
        const uint32_t* src = reinterpret_cast<const uint32_t*>(packed + r * kKvBytes + 12 * l8);
        w[0] = __ldg(src);
        w[1] = __ldg(src + 1);
        w[2] = __ldg(src + 2);
        sc = half_bits_to_float(__ldg(norms + r)) * (1.0f / 256.0f);
      }
#pragma unroll
      for (int e = 0; e < 32; ++e) c[e] = cb[kv_code(w, e)];
    }
    for (int m = 0; m < m_count; ++m) {
      const float4* qm = reinterpret_cast<const float4*>(qs + kv_qpos(m, 32 * l8));
      float acc = 0.0f;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const float4 t = qm[i];
        acc = fmaf(c[4 * i], t.x, acc);
        acc = fmaf(c[4 * i + 1], t.y, acc);
        acc = fmaf(c[4 * i + 2], t.z, acc);
        acc = fmaf(c[4 * i + 3], t.w, acc);
      }
      acc = oct_sum(acc);
      if (active && l8 == 0) S[static_cast<int64_t>(m) * lds + r] = acc * sc;
    }
  }
}

}  // namespace

int launch_kv_quantize(const uint16_t* X, int64_t n, int64_t ldx, const float* codebook, uint8_t* packed,
                       uint16_t* norms, cudaStream_t stream) {
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 4;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(n, kKvThreads / 8)));
  const int xvec = (reinterpret_cast<uintptr_t>(X) % 16 == 0 && (ldx * 2) % 16 == 0) ? 1 : 0;
  kv_quantize_kernel<<<grid, kKvThreads, 0, stream>>>(X, n, ldx, codebook, packed, norms, xvec);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_kv_dequantize(const uint8_t* packed, const uint16_t* norms, const float* codebook, int64_t n, void* out,
                         bool bf16, cudaStream_t stream) {
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 8;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(n, kKvThreads / 8)));
  if (bf16) kv_dequantize_kernel<true><<<grid, kKvThreads, 0, stream>>>(packed, norms, codebook, n, out);
  else kv_dequantize_kernel<false><<<grid, kKvThreads, 0, stream>>>(packed, norms, codebook, n, out);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

int launch_kv_scores(const uint16_t* Q, int64_t m, int64_t ldq, const uint8_t* packed, const uint16_t* norms,
                     const float* codebook, int64_t n_enc, const uint16_t* window, int64_t R, int64_t n_total,
                     float* S, int64_t lds, cudaStream_t stream) {
  const int smem = static_cast<int>(m) * kKvQRow * 4;
  static PerDeviceOnce attr;
  if (const int st = attr([&] {
        return cudaFuncSetAttribute(kv_scores_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                    kKvMaxQueries * kKvQRow * 4) == cudaSuccess;
      }))
    return st;
  const int64_t max_ctas = static_cast<int64_t>(sm_count()) * 4;
  const int grid = static_cast<int>(std::min<int64_t>(max_ctas, ceil_div(n_total, kKvThreads / 8)));
  kv_scores_kernel<<<grid, kKvThreads, smem, stream>>>(Q, static_cast<int>(m), ldq, packed, norms, codebook, n_enc,
                                                       window, R > 0 ? R : 1, n_total, S, lds);
  return cudaGetLastError() == cudaSuccess ? HLWQ_OK : HLWQ_ECUDA;
}

// Appends t tokens to a cache of n_enc encoded tokens and a residual window
// (ring of R slots) holding tokens n_enc .. n_total - 1: the tokens that leave
// the window (oldest first) are encoded into rows n_enc .. n_enc2 - 1, then
// the new tokens that stay are copied into their slots.  Stream order keeps
// every window slot read (encoded) before it is overwritten: a new token that
// stays in slot i % R replaces token i - R, which always leaves.
int launch_kv_window_append(const uint16_t* X, int64_t t, int64_t ldx, uint16_t* window, int64_t R, int64_t n_enc,
                            int64_t n_total, const float* codebook, uint8_t* packed, uint16_t* norms,
                            int64_t* n_enc_out, cudaStream_t stream) {
  const int64_t n_total2 = n_total + t;
  const int64_t n_enc2 = std::max(n_enc, n_total2 - R);
  // old window tokens that leave: [n_enc, min(n_enc2, n_total)), in ring segments
  for (int64_t i = n_enc; i < std::min(n_enc2, n_total);) {
    const int64_t slot = i % R;
    const int64_t cnt = std::min(std::min(n_enc2, n_total) - i, R - slot);
    const int st = launch_kv_quantize(window + slot * kKvDim, cnt, kKvDim, codebook, packed + i * kKvBytes,
                                      norms + i, stream);
    if (st != HLWQ_OK) return st;
    i += cnt;
  }
  // new tokens that leave at once: [max(n_total, n_enc), n_enc2)
  const int64_t d0 = std::max(n_total, n_enc);
  if (n_enc2 > d0) {
    const int st = launch_kv_quantize(X + (d0 - n_total) * ldx, n_enc2 - d0, ldx, codebook, packed + d0 * kKvBytes,
                                      norms + d0, stream);
    if (st != HLWQ_OK) return st;
  }
  // new tokens that stay: [max(n_total, n_enc2), n_total2), in ring segments
  for (int64_t i = std::max(n_total, n_enc2); i < n_total2;) {
    const int64_t slot = i % R;
    const int64_t cnt = std::min(n_total2 - i, R - slot);
    if (cudaMemcpy2DAsync(window + slot * kKvDim, kKvDim * 2, X + (i - n_total) * ldx, ldx * 2, kKvDim * 2,
                          cnt, cudaMemcpyDeviceToDevice, stream) != cudaSuccess)
      return HLWQ_ECUDA;
    i += cnt;
  }
  if (n_enc_out) *n_enc_out = n_enc2;
  return HLWQ_OK;
}

}  // namespace hlwq
